// Decoder attention for bf16 storage: the window self-attention over the
// ring cache C^D and the cross-attention over the memory prefix M_{<=t}
// (jiphyeonjeon review "Recurrent Looped Transformer" §2-§3.3; greeksharifa
// §2.5); also the encoder's causal attention over its cache prefix.  All are
// HBM streams: each (sequence, head) reads its keys and values once.
//
// One CTA per (sequence, head, group of up to NQ query positions), 4 warps.
// The keys of the group live in one contiguous run per head: the memory or
// encoder-cache prefix 1..t, or the ring's occupied slots 0..min(pd, W-1)-1.
// Thread 0 streams the run through a 2-stage shared-memory pipeline with 1-D
// bulk copies (64 keys of K and of V per stage, completion counted on an
// mbarrier); each warp scores its quarter of a stage (d_h/8 lanes per key,
// 16 bytes each), keeps an online softmax per query, and the warps' partial
// results are merged in warp order at the end.  The window's keys of the
// current block (at most NQ positions past the ring) are read directly.
// Key order and every reduction order depend on positions only, so a row's
// result does not depend on the batch.  Waits are bounded.
#include <math.h>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {

__device__ int g_attn_error;   // sticky: a bounded wait of these kernels gave up

int read_and_clear_attn_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        int z = 0;
        cudaMemcpyToSymbol(g_attn_error, &z, sizeof(int));
    }
    return v;
}

namespace {

constexpr int NW = 4;      // warps per CTA
constexpr int CH = 64;     // keys per pipeline stage

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ float slab_sum(const float* __restrict__ P, int S, size_t slab,
                                          size_t i) {
    float v = P[i];
    for (int z = 1; z < S; ++z) v += P[(size_t)z * slab + i];
    return v;
}
// rotate-half RoPE of one pair (j, j + d_h/2)
__device__ __forceinline__ void rope_rot(float x1, float x2, float c, float s, float& y1,
                                         float& y2) {
    y1 = x1 * c - x2 * s;
    y2 = x2 * c + x1 * s;
}

template <int DH, int NQ>
struct Online {             // per-warp online softmax state of NQ queries
    float m[NQ], l[NQ], acc[NQ][8];
};

// Score keys (LPK lanes each; key index from `key_of`) and fold them into the
// state: KPR keys per round, `rounds` rounds, all scores first, then one max /
// rescale, then the value accumulation.
template <int DH, int NQ, int ROUNDS, typename KP, typename VP, typename POS>
__device__ __forceinline__ void fold_keys(Online<DH, NQ>& st, const float (&q)[NQ][8],
                                          const int (&lo)[NQ], const int (&hi)[NQ], KP kptr,
                                          VP vptr, POS pos_of, int lane) {
    constexpr int LPK = DH / 8, KPR = 32 / LPK;
    const int seg = lane % LPK, grp = lane / LPK;
    float s[NQ][ROUNDS];
#pragma unroll
    for (int rr = 0; rr < ROUNDS; ++rr) {
        const int kidx = rr * KPR + grp;
        const int p = pos_of(kidx);            // 0 when the key does not exist
        float kf[8] = {};
        if (p > 0) unpack8(*reinterpret_cast<const uint4*>(kptr(kidx) + seg * 8), kf);
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            float dot = 0.f;
#pragma unroll
            for (int x = 0; x < 8; ++x) dot = fmaf(q[i][x], kf[x], dot);
#pragma unroll
            for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            s[i][rr] = (p > 0 && p >= lo[i] && p <= hi[i]) ? dot : -INFINITY;
        }
    }
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        float bm = s[i][0];
#pragma unroll
        for (int rr = 1; rr < ROUNDS; ++rr) bm = fmaxf(bm, s[i][rr]);
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        const float mn = fmaxf(st.m[i], bm);
        if (mn == -INFINITY) continue;
        const float corr = (st.m[i] == -INFINITY) ? 0.f : expf(st.m[i] - mn);
        float ps = 0.f;
#pragma unroll
        for (int rr = 0; rr < ROUNDS; ++rr) {
            s[i][rr] = (s[i][rr] == -INFINITY) ? 0.f : expf(s[i][rr] - mn);
            ps += s[i][rr];
        }
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        st.l[i] = st.l[i] * corr + ps;
#pragma unroll
        for (int x = 0; x < 8; ++x) st.acc[i][x] *= corr;
        st.m[i] = mn;
    }
#pragma unroll
    for (int rr = 0; rr < ROUNDS; ++rr) {
        const int kidx = rr * KPR + grp;
        if (pos_of(kidx) <= 0) continue;
        float vf[8];
        unpack8(*reinterpret_cast<const uint4*>(vptr(kidx) + seg * 8), vf);
#pragma unroll
        for (int i = 0; i < NQ; ++i)
#pragma unroll
            for (int x = 0; x < 8; ++x) st.acc[i][x] = fmaf(s[i][rr], vf[x], st.acc[i][x]);
    }
}

template <int DH, int NQ, bool SWA, bool PRO>
__global__ void __launch_bounds__(NW * 32)
k_attn_stream(const float* __restrict__ Q, const bf16* __restrict__ base, size_t row_stride,
              int span, const bf16* __restrict__ Kc, const bf16* __restrict__ Vc,
              const int32_t* __restrict__ pos, int W, bf16* __restrict__ A, int n, int heads,
              ProjIn pin) {
    pdl_enter();
    int* err = &g_attn_error;
    constexpr int LPK = DH / 8, KPR = 32 / LPK;
    constexpr int WK = CH / NW;                 // keys per warp per stage
    constexpr int ROUNDS = WK / KPR;
    constexpr uint32_t STAGE_BYTES = CH * DH * 2;
    extern __shared__ __align__(128) uint8_t smem[];
    bf16* sK = reinterpret_cast<bf16*>(smem);                  // [2][CH][DH]
    bf16* sV = reinterpret_cast<bf16*>(smem + 2 * STAGE_BYTES);
    __shared__ uint64_t full[2], empty[2];
    __shared__ float s_m[NW][NQ], s_l[NW][NQ];
    __shared__ float s_o[NW][NQ][DH];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
    const int q0 = blockIdx.y * NQ;
    const int nq = min(NQ, n - q0);
    const int d = heads * DH;
    const int pd = pos[b];
    const int seg = lane % LPK;

    // PRO: q (and, for the window attention, this block's own k and v) are
    // formed here from the projection's partial slabs: summed in slab order,
    // RoPE at the query's position, k and v rounded to the storage type.
    __shared__ __align__(16) float s_q[PRO ? NQ : 1][DH];
    __shared__ __align__(16) bf16 s_k[PRO && SWA ? NQ : 1][DH];
    __shared__ __align__(16) bf16 s_v[PRO && SWA ? NQ : 1][DH];
    if (PRO) {
        constexpr int HALF = DH / 2;
        for (int e = threadIdx.x; e < nq * HALF; e += NW * 32) {
            const int i = e / HALF, j = e % HALF;
            const int t = pd + 1 + q0 + i;
            const float c = pin.rope.cs[(size_t)t * HALF + j], sn = pin.rope.sn[(size_t)t * HALF + j];
            const size_t rb = (size_t)(b * n + q0 + i) * pin.ldp + h * DH + j;
            float y1, y2;
            rope_rot(slab_sum(pin.P, pin.S, pin.slab, rb), slab_sum(pin.P, pin.S, pin.slab, rb + HALF),
                     c, sn, y1, y2);
            s_q[i][j] = y1;
            s_q[i][j + HALF] = y2;
            if (SWA) {
                rope_rot(slab_sum(pin.P, pin.S, pin.slab, rb + d),
                         slab_sum(pin.P, pin.S, pin.slab, rb + d + HALF), c, sn, y1, y2);
                s_k[i][j] = __float2bfloat16_rn(y1);
                s_k[i][j + HALF] = __float2bfloat16_rn(y2);
                s_v[i][j] = __float2bfloat16_rn(slab_sum(pin.P, pin.S, pin.slab, rb + 2 * d));
                s_v[i][j + HALF] =
                    __float2bfloat16_rn(slab_sum(pin.P, pin.S, pin.slab, rb + 2 * d + HALF));
            }
        }
        __syncthreads();
    }

    int lo[NQ], hi[NQ];
    float q[NQ][8];
    const float sc = 1.0f / sqrtf((float)DH);
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const int t = pd + 1 + q0 + min(i, nq - 1);
        hi[i] = i < nq ? t : 0;
        lo[i] = SWA ? max(1, t - W + 1) : 1;
        const float* qp = PRO ? &s_q[min(i, nq - 1)][seg * 8]
                              : Q + (size_t)(b * n + q0 + min(i, nq - 1)) * d + h * DH + seg * 8;
#pragma unroll
        for (int x = 0; x < 8; ++x) q[i][x] = qp[x] * sc;
    }

    // the contiguous run: prefix 1..t_last, or the occupied ring slots
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH;
    const bf16* vg = kg + (size_t)heads * span * DH;
    const int nreg = SWA ? (W > 1 ? min(pd, span) : 0) : hi[nq - 1];
    const int nch = (nreg + CH - 1) / CH;

    if (threadIdx.x == 0) {
        tc::mbar_init(&full[0], 1);
        tc::mbar_init(&full[1], 1);
        tc::mbar_init(&empty[0], NW);
        tc::mbar_init(&empty[1], NW);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    auto issue = [&](int c) {
        const int st = c & 1, k0 = c * CH, cnt = min(CH, nreg - k0);
        const uint32_t bytes = (uint32_t)cnt * DH * 2;
        tc::mbar_expect_tx(&full[st], 2 * bytes);
        bulk_load(sK + (size_t)st * CH * DH, kg + (size_t)k0 * DH, bytes, &full[st]);
        bulk_load(sV + (size_t)st * CH * DH, vg + (size_t)k0 * DH, bytes, &full[st]);
    };
    if (threadIdx.x == 0 && nch > 0) issue(0);

    Online<DH, NQ> os;
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        os.m[i] = -INFINITY;
        os.l[i] = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) os.acc[i][x] = 0.f;
    }
    for (int c = 0; c < nch; ++c) {
        const int st = c & 1;
        if (threadIdx.x == 0 && c + 1 < nch) {
            // stage (c+1)&1 was read by chunk c-1: every warp must be done with it
            if (c >= 1 && !tc::mbar_wait(&empty[(c + 1) & 1], (uint32_t)((c - 1) >> 1) & 1u)) {
                s_abort = 1;
                atomicExch(err, kDevTimeout);
            } else {
                issue(c + 1);
            }
        }
        if (!tc::mbar_wait(&full[st], (uint32_t)(c >> 1) & 1u)) {
            s_abort = 1;
            atomicExch(err, kDevTimeout);
            break;
        }
        const int k0 = c * CH + warp * WK;     // this warp's first key (index in the run)
        const bf16* sk = sK + (size_t)st * CH * DH + (size_t)warp * WK * DH;
        const bf16* sv = sV + (size_t)st * CH * DH + (size_t)warp * WK * DH;
        auto pos_of = [&](int kidx) -> int {
            const int j = k0 + kidx;
            if (j >= nreg) return 0;
            if (!SWA) return j + 1;
            return pd - ((pd - 1 - j) % span);   // ring slot j holds this position
        };
        fold_keys<DH, NQ, ROUNDS>(os, q, lo, hi, [&](int kidx) { return sk + (size_t)kidx * DH; },
                                  [&](int kidx) { return sv + (size_t)kidx * DH; }, pos_of, lane);
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[st]);
        if (s_abort) break;
    }
    if (SWA && warp == 0) {   // the block's own positions pd+1 .. pd+q0+nq (this layer's k, v)
        // (with PRO the grid has one query group, so all of them are in s_k / s_v)
        const bf16* ck = PRO ? &s_k[0][0] : Kc + (size_t)b * n * d + h * DH;
        const bf16* cv = PRO ? &s_v[0][0] : Vc + (size_t)b * n * d + h * DH;
        const int ld = PRO ? DH : d;
        const int nown = q0 + nq;
        for (int e0 = 0; e0 < nown; e0 += KPR) {
            fold_keys<DH, NQ, 1>(
                os, q, lo, hi, [&](int kidx) { return ck + (size_t)(e0 + kidx) * ld; },
                [&](int kidx) { return cv + (size_t)(e0 + kidx) * ld; },
                [&](int kidx) -> int { return e0 + kidx < nown ? pd + 1 + e0 + kidx : 0; }, lane);
        }
    }
    // reduce over the key groups of the warp, then merge the warps in order
#pragma unroll
    for (int i = 0; i < NQ; ++i)
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1)
                os.acc[i][x] += __shfl_xor_sync(0xffffffffu, os.acc[i][x], o);
    if (lane < LPK) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
#pragma unroll
            for (int x = 0; x < 8; ++x) s_o[warp][i][seg * 8 + x] = os.acc[i][x];
            if (lane == 0) {
                s_m[warp][i] = os.m[i];
                s_l[warp][i] = os.l[i];
            }
        }
    }
    __syncthreads();
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
    if (PRO && SWA && W > 1 && !s_abort) {
        // every read of this head's ring has landed (all stages were waited
        // for): move the block's last min(n, W-1) positions into their slots
        const int slots = span;
        bf16* rk = const_cast<bf16*>(kg);
        bf16* rv = const_cast<bf16*>(vg);
        for (int e = threadIdx.x; e < nq * DH; e += NW * 32) {
            const int i = e / DH, x = e % DH;
            if (i < n - slots) continue;
            const int slot = (pd + i) % slots;     // position pd+1+i
            rk[(size_t)slot * DH + x] = s_k[i][x];
            rv[(size_t)slot * DH + x] = s_v[i][x];
        }
    }
}

// One launcher per kernel instance, so that each instance gets its own
// shared-memory attribute (the instances share a function-pointer type).
template <int DH, int NQ, bool SWA, bool PRO>
bool launch_one(const float* Q, const bf16* base, size_t row_stride, int span, const bf16* Kc,
                const bf16* Vc, const int32_t* pos, int W, bf16* A, int B, int n, int heads,
                const ProjIn& pin, cudaStream_t st) {
    constexpr size_t smem = 4 * (size_t)CH * DH * 2;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(k_attn_stream<DH, NQ, SWA, PRO>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return false;
        attr = true;
    }
    launch(k_attn_stream<DH, NQ, SWA, PRO>, dim3(B * heads, (n + NQ - 1) / NQ), NW * 32, smem, st,
           Q, base, row_stride, span, Kc, Vc, pos, W, A, n, heads, pin);
    rlt_count_launch();
    return true;
}

template <int DH, bool SWA, bool PRO>
bool launch_stream(const float* Q, const bf16* base, size_t row_stride, int span, const bf16* Kc,
                   const bf16* Vc, const int32_t* pos, int W, bf16* A, int B, int n, int heads,
                   const ProjIn& pin, cudaStream_t st) {
    if (n == 1)
        return launch_one<DH, 1, SWA, PRO>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B, n,
                                           heads, pin, st);
    if (n == 2)
        return launch_one<DH, 2, SWA, PRO>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B, n,
                                           heads, pin, st);
    return launch_one<DH, 4, SWA, PRO>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B, n, heads,
                                       pin, st);
}

}  // namespace

// bf16 attention with head size 64 or 128; returns false otherwise.
bool launch_attn_cross_fast(const float* Q, const bf16* mem, size_t row_stride, int T_cap,
                            const int32_t* pos, bf16* A, int B, int n, int heads, int dh,
                            cudaStream_t st) {
    if (B * n <= 0) return true;
    if (dh == 64)
        return launch_stream<64, false, false>(Q, mem, row_stride, T_cap, nullptr, nullptr, pos, 0,
                                               A, B, n, heads, ProjIn{}, st);
    if (dh == 128)
        return launch_stream<128, false, false>(Q, mem, row_stride, T_cap, nullptr, nullptr, pos,
                                                0, A, B, n, heads, ProjIn{}, st);
    return false;
}

bool launch_attn_swa_fast(const float* Q, const bf16* Kc, const bf16* Vc, const bf16* ring,
                          size_t row_stride, int W, const int32_t* pos, bf16* A, int B, int n,
                          int heads, int dh, cudaStream_t st) {
    if (B * n <= 0) return true;
    const int slots = W > 1 ? W - 1 : 1;
    if (dh == 64)
        return launch_stream<64, true, false>(Q, ring, row_stride, slots, Kc, Vc, pos, W, A, B, n,
                                              heads, ProjIn{}, st);
    if (dh == 128)
        return launch_stream<128, true, false>(Q, ring, row_stride, slots, Kc, Vc, pos, W, A, B,
                                               n, heads, ProjIn{}, st);
    return false;
}

bool launch_attn_swa_proj(const ProjIn& pin, bf16* ring, size_t row_stride, int W,
                          const int32_t* pos, bf16* A, int B, int n, int heads, int dh,
                          cudaStream_t st) {
    // one query group per (sequence, head): the kernel then owns every read
    // and write of that head's ring for the block
    if (!fast_attn_enabled() || n > 4 || (dh != 64 && dh != 128)) return false;
    if (B * n <= 0) return true;
    const int slots = W > 1 ? W - 1 : 1;
    if (dh == 64)
        return launch_stream<64, true, true>(nullptr, ring, row_stride, slots, nullptr, nullptr,
                                             pos, W, A, B, n, heads, pin, st);
    return launch_stream<128, true, true>(nullptr, ring, row_stride, slots, nullptr, nullptr, pos,
                                          W, A, B, n, heads, pin, st);
}

bool launch_attn_cross_proj(const ProjIn& pin, const bf16* mem, size_t row_stride, int T_cap,
                            const int32_t* pos, bf16* A, int B, int n, int heads, int dh,
                            cudaStream_t st) {
    if (!fast_attn_enabled() || (dh != 64 && dh != 128)) return false;
    if (B * n <= 0) return true;
    if (dh == 64)
        return launch_stream<64, false, true>(nullptr, mem, row_stride, T_cap, nullptr, nullptr,
                                              pos, 0, A, B, n, heads, pin, st);
    return launch_stream<128, false, true>(nullptr, mem, row_stride, T_cap, nullptr, nullptr, pos,
                                           0, A, B, n, heads, pin, st);
}

}  // namespace rlt
