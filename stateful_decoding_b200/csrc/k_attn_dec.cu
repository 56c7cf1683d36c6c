// Decoder attention for bf16 storage: the window self-attention over the
// ring cache C^D and the cross-attention over the memory prefix M_{<=t}
// (jiphyeonjeon review "Recurrent Looped Transformer" §2-§3.3; greeksharifa
// §2.5).  Both are HBM streams: each (sequence, head) reads its keys and
// values once per call.
//
// One CTA per (sequence, head, group of up to NQ query positions).  The keys
// of the union of the group's windows are split into blocks of 8*KPL keys,
// dealt round-robin to 4 warps.  Inside a warp, LPK = DH/8 lanes share one
// key: each lane loads 16 bytes (8 values) of it, so one warp-wide load
// brings KPL whole keys; a score is a lane-group dot product reduced with
// shuffles.  Each warp keeps an online softmax per query; the warps' partial
// (max, sum, output) are merged in shared memory in warp order.  Key order
// and reduction order depend only on the positions, never on the batch.
#include <math.h>

#include "kernels.cuh"

namespace rlt {

namespace {

constexpr int NW = 4;   // warps per CTA

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

template <int DH, int NQ, bool SWA>
__global__ void __launch_bounds__(NW * 32)
k_attn_dec(const float* __restrict__ Q, const bf16* __restrict__ base, size_t row_stride,
           int span,                          // cross: T_cap; window: W-1 ring slots
           const bf16* __restrict__ Kc, const bf16* __restrict__ Vc,
           const int32_t* __restrict__ pos_dec, int W, bf16* __restrict__ A, int n, int heads) {
    constexpr int LPK = DH / 8;          // lanes per key
    constexpr int KPL = 32 / LPK;        // keys per warp-wide load
    constexpr int BLK = 8 * KPL;         // keys per block (8 loads per lane)
    __shared__ float s_m[NW][NQ], s_l[NW][NQ];
    __shared__ float s_o[NW][NQ][DH];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
    const int q0 = blockIdx.y * NQ;
    const int nq = min(NQ, n - q0);
    const int d = heads * DH;
    const int pd = pos_dec[b];
    const int seg = lane % LPK, grp = lane / LPK;

    // key sources
    const bf16* kb = base + (size_t)b * row_stride + (size_t)h * span * DH;
    const bf16* vb = kb + (size_t)heads * span * DH;
    const bf16* ck = Kc + (size_t)b * n * d + h * DH;
    const bf16* cv = Vc + (size_t)b * n * d + h * DH;

    // query windows: query i at t_i = pd + 1 + q0 + i
    int lo[NQ], hi[NQ];
    float q[NQ][8];
    const float sc = 1.0f / sqrtf((float)DH);
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const int t = pd + 1 + q0 + min(i, nq - 1);
        hi[i] = i < nq ? t : 0;
        lo[i] = SWA ? max(1, t - W + 1) : 1;
        const float* qp = Q + (size_t)(b * n + q0 + min(i, nq - 1)) * d + h * DH + seg * 8;
#pragma unroll
        for (int x = 0; x < 8; ++x) q[i][x] = qp[x] * sc;
    }
    const int u_lo = lo[0], u_hi = hi[nq - 1];     // union of the windows
    const int nkeys = u_hi - u_lo + 1;

    auto kaddr = [&](int p, bool val) -> const bf16* {
        if (!SWA) return (val ? vb : kb) + (size_t)(p - 1) * DH;
        if (p <= pd) return (val ? vb : kb) + (size_t)((p - 1) % span) * DH;
        return (val ? cv : ck) + (size_t)(p - pd - 1) * d;
    };

    float m[NQ], l[NQ], acc[NQ][8];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[i][x] = 0.f;
    }

    for (int blk = warp; blk * BLK < nkeys; blk += NW) {
        const int p0 = u_lo + blk * BLK;
        uint4 kr[8], vr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int p = p0 + j * KPL + grp;
            if (p <= u_hi) {
                kr[j] = *reinterpret_cast<const uint4*>(kaddr(p, false) + seg * 8);
                vr[j] = *reinterpret_cast<const uint4*>(kaddr(p, true) + seg * 8);
            } else {
                kr[j] = make_uint4(0, 0, 0, 0);
                vr[j] = make_uint4(0, 0, 0, 0);
            }
        }
        float s[NQ][8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float kf[8];
            bf16x8_to_f32(kr[j], kf);
            const int p = p0 + j * KPL + grp;
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                float dot = 0.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) dot = fmaf(q[i][x], kf[x], dot);
#pragma unroll
                for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                s[i][j] = (p >= lo[i] && p <= hi[i]) ? dot : -INFINITY;
            }
        }
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            float bm = s[i][0];
#pragma unroll
            for (int j = 1; j < 8; ++j) bm = fmaxf(bm, s[i][j]);
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const float mn = fmaxf(m[i], bm);
            if (mn == -INFINITY) continue;          // nothing of this query in the block yet
            const float corr = (m[i] == -INFINITY) ? 0.f : expf(m[i] - mn);
            float ps = 0.f, pj[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                pj[j] = (s[i][j] == -INFINITY) ? 0.f : expf(s[i][j] - mn);
                ps += pj[j];
            }
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l[i] = l[i] * corr + ps;
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[i][x] *= corr;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float vf[8];
                bf16x8_to_f32(vr[j], vf);
#pragma unroll
                for (int x = 0; x < 8; ++x) acc[i][x] = fmaf(pj[j], vf[x], acc[i][x]);
            }
            m[i] = mn;
        }
    }
    // reduce the partial outputs over the key groups of the warp
#pragma unroll
    for (int i = 0; i < NQ; ++i)
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1)
                acc[i][x] += __shfl_xor_sync(0xffffffffu, acc[i][x], o);
    if (lane < LPK) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
#pragma unroll
            for (int x = 0; x < 8; ++x) s_o[warp][i][seg * 8 + x] = acc[i][x];
            if (lane == 0) {
                s_m[warp][i] = m[i];
                s_l[warp][i] = l[i];
            }
        }
    }
    __syncthreads();
    // merge the warps in order; thread x of the CTA owns output dim x of each query
    for (int e = threadIdx.x; e < nq * DH; e += NW * 32) {
        const int i = e / DH, x = e % DH;
        float M = -INFINITY;
        for (int w = 0; w < NW; ++w) M = fmaxf(M, s_m[w][i]);
        float L = 0.f, O = 0.f;
        for (int w = 0; w < NW; ++w) {
            if (s_m[w][i] == -INFINITY) continue;
            const float f = expf(s_m[w][i] - M);
            L += s_l[w][i] * f;
            O += s_o[w][i][x] * f;
        }
        A[(size_t)(b * n + q0 + i) * d + h * DH + x] = __float2bfloat16_rn(O / L);
    }
}

template <int DH, bool SWA>
void launch_dec(const float* Q, const bf16* base, size_t row_stride, int span, const bf16* Kc,
                const bf16* Vc, const int32_t* pos_dec, int W, bf16* A, int B, int n, int heads,
                cudaStream_t st) {
    if (n == 1) {
        k_attn_dec<DH, 1, SWA><<<dim3(B * heads, 1), NW * 32, 0, st>>>(
            Q, base, row_stride, span, Kc, Vc, pos_dec, W, A, n, heads);
    } else if (n == 2) {
        k_attn_dec<DH, 2, SWA><<<dim3(B * heads, 1), NW * 32, 0, st>>>(
            Q, base, row_stride, span, Kc, Vc, pos_dec, W, A, n, heads);
    } else {
        k_attn_dec<DH, 4, SWA><<<dim3(B * heads, (n + 3) / 4), NW * 32, 0, st>>>(
            Q, base, row_stride, span, Kc, Vc, pos_dec, W, A, n, heads);
    }
    rlt_count_launch();
}

}  // namespace

// bf16 decoder attention with head size 64 or 128; returns false otherwise.
bool launch_attn_cross_fast(const float* Q, const bf16* mem, size_t row_stride, int T_cap,
                            const int32_t* pos_dec, bf16* A, int B, int n, int heads, int dh,
                            cudaStream_t st) {
    if (B * n <= 0) return true;
    if (dh == 64) launch_dec<64, false>(Q, mem, row_stride, T_cap, nullptr, nullptr, pos_dec, 0, A, B, n, heads, st);
    else if (dh == 128) launch_dec<128, false>(Q, mem, row_stride, T_cap, nullptr, nullptr, pos_dec, 0, A, B, n, heads, st);
    else return false;
    return true;
}

bool launch_attn_swa_fast(const float* Q, const bf16* Kc, const bf16* Vc, const bf16* ring,
                          size_t row_stride, int W, const int32_t* pos_dec, bf16* A, int B, int n,
                          int heads, int dh, cudaStream_t st) {
    if (B * n <= 0) return true;
    const int slots = W > 1 ? W - 1 : 1;
    if (dh == 64) launch_dec<64, true>(Q, ring, row_stride, slots, Kc, Vc, pos_dec, W, A, B, n, heads, st);
    else if (dh == 128) launch_dec<128, true>(Q, ring, row_stride, slots, Kc, Vc, pos_dec, W, A, B, n, heads, st);
    else return false;
    return true;
}

}  // namespace rlt
