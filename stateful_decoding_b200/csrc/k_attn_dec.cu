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

#include <algorithm>
#include <cstdlib>
#include <cstring>

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

// Sum of S (<= 8) split-K partial slabs at element i, in slab order; all
// loads are issued before the first add.
__device__ __forceinline__ float slab_sum8(const float* __restrict__ P, int S, size_t slab,
                                           size_t i) {
    float t[8];
#pragma unroll
    for (int z = 0; z < 8; ++z)
        if (z < S) t[z] = P[(size_t)z * slab + i];
    float v = t[0];
#pragma unroll
    for (int z = 1; z < 8; ++z)
        if (z < S) v += t[z];
    return v;
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

template <int DH, int NQ, bool SWA, bool PRO, int NSTG>
__global__ void __launch_bounds__(NW * 32)
k_attn_stream(const float* __restrict__ Q, const bf16* __restrict__ base, size_t row_stride,
              int span, const bf16* __restrict__ Kc, const bf16* __restrict__ Vc,
              const int32_t* __restrict__ pos, int W, bf16* __restrict__ A, int n, int heads,
              ProjIn pin) {
    // Decoder launches (PRO) start streaming keys before waiting for the
    // previous kernel: the ring and the memory were last written two or more
    // kernels back, and the position counter is read through L2.  Only q and
    // the block's own k, v come from the kernel just before.
    if (!PRO) pdl_enter();
    int* err = &g_attn_error;
    constexpr int LPK = DH / 8, KPR = 32 / LPK;
    constexpr int WK = CH / NW;                 // keys per warp per stage
    constexpr int ROUNDS = WK / KPR;
    constexpr uint32_t STAGE_BYTES = CH * DH * 2;
    extern __shared__ __align__(128) uint8_t smem[];
    bf16* sK = reinterpret_cast<bf16*>(smem);                  // [NSTG][CH][DH]
    bf16* sV = reinterpret_cast<bf16*>(smem + NSTG * STAGE_BYTES);
    __shared__ uint64_t full[2], empty[2];
    __shared__ float s_m[NW][NQ], s_l[NW][NQ];
    __shared__ float s_o[NW][NQ][DH];
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
    const int q0 = blockIdx.y * NQ;
    const int nq = min(NQ, n - q0);
    const int d = heads * DH;
    const int pd = PRO ? __ldcg(pos + b) : pos[b];
    const int seg = lane % LPK;

    // the contiguous run: prefix 1..t_last, or the occupied ring slots
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH;
    const bf16* vg = kg + (size_t)heads * span * DH;
    const int nreg = SWA ? (W > 1 ? min(pd, span) : 0) : pd + q0 + nq;
    const int nch = (nreg + CH - 1) / CH;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NSTG; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], NW);
        }
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    int nissued = 0;                         // chunks issued (thread 0)
    auto issue = [&](int c) {
        const int st = c % NSTG, k0 = c * CH, cnt = min(CH, nreg - k0);
        const uint32_t bytes = (uint32_t)cnt * DH * 2;
        tc::mbar_expect_tx(&full[st], 2 * bytes);
        bulk_load(sK + (size_t)st * CH * DH, kg + (size_t)k0 * DH, bytes, &full[st]);
        bulk_load(sV + (size_t)st * CH * DH, vg + (size_t)k0 * DH, bytes, &full[st]);
        nissued = c + 1;
    };
    // every stage starts empty: fill them all before anything else
    if (threadIdx.x == 0)
        for (int c = 0; c < min(nch, NSTG); ++c) issue(c);
    if (PRO) pdl_enter();

    // PRO: q (and, for the window attention, this block's own k and v) are
    // formed here from the projection's partial slabs: summed in slab order,
    // RoPE at the query's position, k and v rounded to the storage type.
    __shared__ __align__(16) float s_q[PRO ? NQ : 1][DH];
    __shared__ __align__(16) bf16 s_k[PRO && SWA ? NQ : 1][DH];
    __shared__ __align__(16) bf16 s_v[PRO && SWA ? NQ : 1][DH];
    if (PRO) {
        // work items per query: HALF rotated q pairs, then (window attention)
        // HALF rotated k pairs and DH v elements; each thread issues all the
        // slab loads of an item before summing them
        constexpr int HALF = DH / 2;
        constexpr int PER = SWA ? 2 * DH : HALF;
        for (int e = threadIdx.x; e < nq * PER; e += NW * 32) {
            const int i = e / PER, r = e % PER;
            const int t = pd + 1 + q0 + i;
            const size_t rb = (size_t)(b * n + q0 + i) * pin.ldp + h * DH;
            if (r < DH) {
                const int j = r % HALF;
                const size_t o = rb + (r < HALF ? 0 : d) + j;     // q pair, or k pair
                const float c = pin.rope.cs[(size_t)t * HALF + j];
                const float sn = pin.rope.sn[(size_t)t * HALF + j];
                float y1, y2;
                rope_pair(slab_sum8(pin.P, pin.S, pin.slab, o),
                         slab_sum8(pin.P, pin.S, pin.slab, o + HALF), c, sn, y1, y2);
                if (r < HALF) {
                    s_q[i][j] = y1;
                    s_q[i][j + HALF] = y2;
                } else {
                    s_k[i][j] = __float2bfloat16_rn(y1);
                    s_k[i][j + HALF] = __float2bfloat16_rn(y2);
                }
            } else {
                const int x = r - DH;
                s_v[i][x] = __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + x));
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

    Online<DH, NQ> os;
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        os.m[i] = -INFINITY;
        os.l[i] = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) os.acc[i][x] = 0.f;
    }
    for (int c = 0; c < nch; ++c) {
        const int st = c % NSTG;
        if (threadIdx.x == 0 && c >= 1 && c - 1 + NSTG < nch) {
            // refill the stage chunk c-1 used, once every warp is done with it
            const int sp = (c - 1) % NSTG;
            if (!tc::mbar_wait(&empty[sp], (uint32_t)((c - 1) / NSTG) & 1u)) {
                s_abort = 1;
                atomicExch(err, kDevTimeout);
            } else {
                issue(c - 1 + NSTG);
            }
        }
        if (!tc::mbar_wait(&full[st], (uint32_t)(c / NSTG) & 1u)) {
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
    if (threadIdx.x == 0 && s_abort) {
        // copies still in flight must land before the CTA exits (bounded)
        for (int i = 0; i < NSTG && i < nissued; ++i) {
            const int last = nissued - 1 - ((nissued - 1 - i) % NSTG);
            tc::mbar_wait(&full[i], (uint32_t)(last / NSTG) & 1u, 1u << 20);
        }
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

// ---------------------------------------------------------------- one-position decode
// Softmax exponentials use the fast exp2-based intrinsic (bf16 storage only).
// One position per row (n = 1, the decode shape): one warp per (row, head),
// four items per CTA, no shared pipeline and no cross-warp merge.  The warp
// forms q (and, for the window attention, the position's own k and v) from
// the projection slabs, then walks the keys in batches of DRB rounds: the K
// and V loads of a batch (16 bytes per lane, d_h/8 lanes per key) are all
// issued before the first is used, then scores, one max and rescale per
// batch, and the value accumulation.  Every occupied ring slot lies inside
// the window and every memory key up to t is visible, so the only mask is
// the run's length.  The keys of the first batch are requested before the
// wait for the previous kernel (ring and memory are written two or more
// kernels back).
constexpr int DWARPS = 4;      // items (warps) per CTA

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// 16 bytes of cached keys/values: kept in L2 (KEEP) or streamed (evict-first)
template <bool KEEP>
__device__ __forceinline__ uint4 ld_kv(const bf16* p, uint64_t pol) {
    if (!KEEP) return __ldcs(reinterpret_cast<const uint4*>(p));
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}
constexpr int DRB = 4;         // rounds per batch (two batches in flight)

template <int DH, bool SWA>
__global__ void __launch_bounds__(DWARPS * 32)
k_attn_dec1(const bf16* __restrict__ base, size_t row_stride, int span,
            const int32_t* __restrict__ pos, int W, bf16* __restrict__ A, int B, int heads,
            ProjIn pin) {
    constexpr int LPK = DH / 8, KPR = 32 / LPK, HALF = DH / 2;
    __shared__ __align__(16) float s_q[DWARPS][DH];
    __shared__ __align__(16) bf16 s_k[DWARPS][DH];
    __shared__ __align__(16) bf16 s_v[DWARPS][DH];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int it = blockIdx.x * DWARPS + warp;
    const bool in_range = it < B * heads;
    const int b = in_range ? it / heads : 0, h = in_range ? it % heads : 0;
    const int d = heads * DH, seg = lane % LPK, grp = lane / LPK;
    const int pd = in_range ? __ldcg(pos + b) : 0, t = pd + 1;
    // debug builds: the position must have rows in the RoPE tables and (for
    // the memory) keys 1..t inside the buffer; the ring slot pd mod (W-1) is
    // then inside the ring.  A failed check skips the item.
    const bool live = in_range && dcheck(pd >= 0 && t <= pin.rope.max_pos && (SWA || t <= span),
                                         &g_attn_error, kDevCapacity);
    const int nreg = !live ? 0 : (SWA ? (W > 1 ? min(pd, span) : 0) : t);
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH + seg * 8;
    const bf16* vg = kg + (size_t)heads * span * DH;

    // The memory is read by every decoder block of the step (one group shared
    // by all blocks): its lines are kept in L2 (evict-last) so that the next
    // blocks' cross-attention can find them there; the window ring, read once
    // per step, streams through (evict-first).
    const uint64_t l2pol = SWA ? 0 : l2_evict_last_policy();
    // two batch buffers: the loads of batch i+1 are in flight while batch i is folded
    uint4 kb0[DRB], vb0[DRB], kb1[DRB], vb1[DRB];
    auto load_batch = [&](int j0, uint4 (&kb)[DRB], uint4 (&vb)[DRB]) {
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            const int j = j0 + r * KPR + grp;
            if (j < nreg) {
                kb[r] = ld_kv<!SWA>(kg + (size_t)j * DH, l2pol);
                vb[r] = ld_kv<!SWA>(vg + (size_t)j * DH, l2pol);
            }
        }
    };
    constexpr int BATCH = DRB * KPR;             // keys per batch
    load_batch(0, kb0, vb0);
    if (BATCH < nreg) load_batch(BATCH, kb1, vb1);
    pdl_enter();

    // q: lane j forms the rotate-half pair (j, j + HALF)
    const size_t rb = (size_t)b * pin.ldp + h * DH;
    const float* cs = pin.rope.cs + (size_t)t * HALF;
    const float* sn = pin.rope.sn + (size_t)t * HALF;
    if (live) {
        for (int j = lane; j < HALF; j += 32) {
            float y1, y2;
            rope_pair(slab_sum8(pin.P, pin.S, pin.slab, rb + j),
                     slab_sum8(pin.P, pin.S, pin.slab, rb + j + HALF), cs[j], sn[j], y1, y2);
            s_q[warp][j] = y1;
            s_q[warp][j + HALF] = y2;
        }
    }
    __syncwarp();
    const float sc = 1.0f / sqrtf((float)DH);
    float q[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) q[x] = s_q[warp][seg * 8 + x] * sc;

    float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) acc[x] = 0.f;
    // fold the batch of keys j0.. held in kb, vb
    auto fold = [&](int j0, const uint4 (&kb)[DRB], const uint4 (&vb)[DRB]) {
        float s[DRB];
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            const bool v = j0 + r * KPR + grp < nreg;
            float kf[8] = {};
            if (v) unpack8(kb[r], kf);
            float dot = 0.f;
#pragma unroll
            for (int x = 0; x < 8; ++x) dot = fmaf(q[x], kf[x], dot);
#pragma unroll
            for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            s[r] = v ? dot : -INFINITY;
        }
        float bm = s[0];
#pragma unroll
        for (int r = 1; r < DRB; ++r) bm = fmaxf(bm, s[r]);
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        const float mn = fmaxf(m, bm);          // finite: the batch holds a key
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        float ps = 0.f;
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            s[r] = (s[r] == -INFINITY) ? 0.f : __expf(s[r] - mn);
            ps += s[r];
        }
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l = l * corr + ps;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] *= corr;
        m = mn;
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            if (!(j0 + r * KPR + grp < nreg)) continue;
            float vf[8];
            unpack8(vb[r], vf);
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = fmaf(s[r], vf[x], acc[x]);
        }
    };
    for (int j0 = 0; j0 < nreg; j0 += 2 * BATCH) {
        fold(j0, kb0, vb0);
        if (j0 + 2 * BATCH < nreg) load_batch(j0 + 2 * BATCH, kb0, vb0);
        if (j0 + BATCH >= nreg) break;
        fold(j0 + BATCH, kb1, vb1);
        if (j0 + 3 * BATCH < nreg) load_batch(j0 + 3 * BATCH, kb1, vb1);
    }
    if (SWA && live) {
        // the current position's own k and v (formed after the loop, when the
        // batch registers are free), rounded like the stored ones
        for (int j = lane; j < HALF; j += 32) {
            float y1, y2;
            rope_pair(slab_sum8(pin.P, pin.S, pin.slab, rb + d + j),
                     slab_sum8(pin.P, pin.S, pin.slab, rb + d + j + HALF), cs[j], sn[j], y1, y2);
            s_k[warp][j] = __float2bfloat16_rn(y1);
            s_k[warp][j + HALF] = __float2bfloat16_rn(y2);
            s_v[warp][j] = __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + j));
            s_v[warp][j + HALF] =
                __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + j + HALF));
        }
        __syncwarp();
        // the current position itself: one key, every lane group scores it,
        // group 0 accumulates its value
        float kf[8], vf[8];
        unpack8(*reinterpret_cast<const uint4*>(&s_k[warp][seg * 8]), kf);
        unpack8(*reinterpret_cast<const uint4*>(&s_v[warp][seg * 8]), vf);
        float dot = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) dot = fmaf(q[x], kf[x], dot);
#pragma unroll
        for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float mn = fmaxf(m, dot);
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        const float p = __expf(dot - mn);
        l = l * corr + p;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] = acc[x] * corr + (grp == 0 ? p * vf[x] : 0.f);
        m = mn;
    }
    // reduce over the key groups; lanes of group 0 hold the head's output
#pragma unroll
    for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) acc[x] += __shfl_xor_sync(0xffffffffu, acc[x], o);
    if (live && grp == 0) {
        const float inv = 1.0f / l;
        uint4 w;
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            __nv_bfloat162 p2 = __floats2bfloat162_rn(acc[2 * x] * inv, acc[2 * x + 1] * inv);
            wp[x] = *reinterpret_cast<uint32_t*>(&p2);
        }
        *reinterpret_cast<uint4*>(A + (size_t)b * d + h * DH + seg * 8) = w;
        if (SWA && W > 1) {
            // all of this head's ring has been read: the position enters slot pd mod (W-1)
            const size_t slot = (size_t)(pd % span) * DH;
            *reinterpret_cast<uint4*>(const_cast<bf16*>(kg) + slot) =
                *reinterpret_cast<const uint4*>(&s_k[warp][seg * 8]);
            *reinterpret_cast<uint4*>(const_cast<bf16*>(vg) + slot) =
                *reinterpret_cast<const uint4*>(&s_v[warp][seg * 8]);
        }
    }
}

// Blocks of NQ = 2..4 positions per row (RLT-2 chunks): one warp per (row,
// head) as in k_attn_dec1, every key scored against all NQ queries of the
// block, an online softmax per query.  The window attention takes the ring's
// keys (query i at t_i = pd+1+i sees positions t_i-W+1 .. t_i, so the oldest
// slots fall out of the later queries' windows), then the block's own
// positions e <= i, formed from the projection slabs after the key loop, and
// finally moves the block's positions into their ring slots -- after every
// read of the ring (the warp owns its (row, head) ring).  The
// cross-attention takes memory keys 1..t_i for query i.  Key order and every
// reduction order depend on positions only.
constexpr int DRBN = 2;        // rounds per batch for multi-query blocks (registers)

template <int DH, bool SWA, int NQ>
__global__ void __launch_bounds__(DWARPS * 32)
k_attn_decn(const bf16* __restrict__ base, size_t row_stride, int span,
            const int32_t* __restrict__ pos, int W, bf16* __restrict__ A, int B, int heads,
            ProjIn pin) {
    constexpr int LPK = DH / 8, KPR = 32 / LPK, HALF = DH / 2;
    constexpr int BATCH = DRBN * KPR;
    __shared__ __align__(16) float s_q[DWARPS][NQ][DH];
    __shared__ __align__(16) bf16 s_k[DWARPS][SWA ? NQ : 1][DH];
    __shared__ __align__(16) bf16 s_v[DWARPS][SWA ? NQ : 1][DH];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int it = blockIdx.x * DWARPS + warp;
    const bool in_range = it < B * heads;
    const int b = in_range ? it / heads : 0, h = in_range ? it % heads : 0;
    const int d = heads * DH, seg = lane % LPK, grp = lane / LPK;
    const int pd = in_range ? __ldcg(pos + b) : 0;
    const bool live = in_range && dcheck(pd >= 0 && pd + NQ <= pin.rope.max_pos &&
                                             (SWA || pd + NQ <= span),
                                         &g_attn_error, kDevCapacity);
    const int nreg = !live ? 0 : (SWA ? (W > 1 ? min(pd, span) : 0) : pd + NQ);
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH + seg * 8;
    const bf16* vg = kg + (size_t)heads * span * DH;
    const uint64_t l2pol = SWA ? 0 : l2_evict_last_policy();
    uint4 kb0[DRBN], vb0[DRBN], kb1[DRBN], vb1[DRBN];
    auto load_batch = [&](int j0, uint4 (&kb)[DRBN], uint4 (&vb)[DRBN]) {
#pragma unroll
        for (int r = 0; r < DRBN; ++r) {
            const int j = j0 + r * KPR + grp;
            if (j < nreg) {
                kb[r] = ld_kv<!SWA>(kg + (size_t)j * DH, l2pol);
                vb[r] = ld_kv<!SWA>(vg + (size_t)j * DH, l2pol);
            }
        }
    };
    load_batch(0, kb0, vb0);
    if (BATCH < nreg) load_batch(BATCH, kb1, vb1);
    pdl_enter();

    // the block's queries: rows b*NQ + i of the slabs, RoPE at t_i
    if (live) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            const size_t rb = (size_t)(b * NQ + i) * pin.ldp + h * DH;
            const float* cs = pin.rope.cs + (size_t)(pd + 1 + i) * HALF;
            const float* sn = pin.rope.sn + (size_t)(pd + 1 + i) * HALF;
            for (int j = lane; j < HALF; j += 32) {
                float y1, y2;
                rope_pair(slab_sum8(pin.P, pin.S, pin.slab, rb + j),
                         slab_sum8(pin.P, pin.S, pin.slab, rb + j + HALF), cs[j], sn[j], y1, y2);
                s_q[warp][i][j] = y1;
                s_q[warp][i][j + HALF] = y2;
            }
        }
    }
    __syncwarp();
    const float sc = 1.0f / sqrtf((float)DH);
    float q[NQ][8];
#pragma unroll
    for (int i = 0; i < NQ; ++i)
#pragma unroll
        for (int x = 0; x < 8; ++x) q[i][x] = s_q[warp][i][seg * 8 + x] * sc;
    float m[NQ], l[NQ], acc[NQ][8];
    int lo[NQ];                      // first visible position of query i
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
        lo[i] = SWA ? max(1, pd + 1 + i - W + 1) : 1;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[i][x] = 0.f;
    }
    // position of run key j: ring slot j holds the newest position <= pd of
    // its residue; memory key j is position j + 1
    auto pos_of = [&](int j) -> int { return SWA ? pd - ((pd - 1 - j) % span) : j + 1; };
    // fold `cnt` keys (their scores per query in s, masked by -inf) into the
    // per-query state; vf: the keys' values
    auto fold = [&](float (&s)[NQ][DRBN], const float (&vf)[DRBN][8], int cnt) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            float bm = s[i][0];
#pragma unroll
            for (int r = 1; r < DRBN; ++r)
                if (r < cnt) bm = fmaxf(bm, s[i][r]);
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            const float mn = fmaxf(m[i], bm);
            if (mn == -INFINITY) continue;            // no visible key yet (warp-uniform)
            const float corr = (m[i] == -INFINITY) ? 0.f : __expf(m[i] - mn);
            float ps = 0.f;
#pragma unroll
            for (int r = 0; r < DRBN; ++r) {
                s[i][r] = (r >= cnt || s[i][r] == -INFINITY) ? 0.f : __expf(s[i][r] - mn);
                ps += s[i][r];
            }
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l[i] = l[i] * corr + ps;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                float a = acc[i][x] * corr;
#pragma unroll
                for (int r = 0; r < DRBN; ++r) a = fmaf(s[i][r], vf[r][x], a);
                acc[i][x] = a;
            }
            m[i] = mn;
        }
    };
    auto fold_batch = [&](int j0, const uint4 (&kb)[DRBN], const uint4 (&vb)[DRBN]) {
        float s[NQ][DRBN], vf[DRBN][8];
#pragma unroll
        for (int r = 0; r < DRBN; ++r) {
            const int j = j0 + r * KPR + grp;
            const bool v = j < nreg;
            const int p = v ? pos_of(j) : 0;
            float kf[8] = {};
            if (v) {
                unpack8(kb[r], kf);
                unpack8(vb[r], vf[r]);
            } else {
#pragma unroll
                for (int x = 0; x < 8; ++x) vf[r][x] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                float dot = 0.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) dot = fmaf(q[i][x], kf[x], dot);
#pragma unroll
                for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                s[i][r] = (v && p >= lo[i] && p <= pd + 1 + i) ? dot : -INFINITY;
            }
        }
        fold(s, vf, DRBN);
    };
    for (int j0 = 0; j0 < nreg; j0 += 2 * BATCH) {
        fold_batch(j0, kb0, vb0);
        if (j0 + 2 * BATCH < nreg) load_batch(j0 + 2 * BATCH, kb0, vb0);
        if (j0 + BATCH >= nreg) break;
        fold_batch(j0 + BATCH, kb1, vb1);
        if (j0 + 3 * BATCH < nreg) load_batch(j0 + 3 * BATCH, kb1, vb1);
    }
    if (SWA && live) {
        // the block's own keys and values, rounded like the stored ones
#pragma unroll
        for (int e = 0; e < NQ; ++e) {
            const size_t rb = (size_t)(b * NQ + e) * pin.ldp + h * DH;
            const float* cs = pin.rope.cs + (size_t)(pd + 1 + e) * HALF;
            const float* sn = pin.rope.sn + (size_t)(pd + 1 + e) * HALF;
            for (int j = lane; j < HALF; j += 32) {
                float y1, y2;
                rope_pair(slab_sum8(pin.P, pin.S, pin.slab, rb + d + j),
                         slab_sum8(pin.P, pin.S, pin.slab, rb + d + j + HALF), cs[j], sn[j], y1,
                         y2);
                s_k[warp][e][j] = __float2bfloat16_rn(y1);
                s_k[warp][e][j + HALF] = __float2bfloat16_rn(y2);
                s_v[warp][e][j] = __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + j));
                s_v[warp][e][j + HALF] =
                    __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + j + HALF));
            }
        }
        __syncwarp();
        // own position e (t_e = pd+1+e): every lane group scores it, group 0
        // carries its value (the others add zeros)
#pragma unroll
        for (int e = 0; e < NQ; ++e) {
            float kf[8], s[NQ][DRBN], vf[DRBN][8];
            unpack8(*reinterpret_cast<const uint4*>(&s_k[warp][e][seg * 8]), kf);
            unpack8(*reinterpret_cast<const uint4*>(&s_v[warp][e][seg * 8]), vf[0]);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                if (grp != 0) vf[0][x] = 0.f;
#pragma unroll
                for (int r = 1; r < DRBN; ++r) vf[r][x] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                float dot = 0.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) dot = fmaf(q[i][x], kf[x], dot);
#pragma unroll
                for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                // one key per lane group would be counted KPR times: only
                // group 0 contributes the score to the block max and the sum
                const bool vis = e <= i && pd + 1 + e >= lo[i];
                s[i][0] = (vis && grp == 0) ? dot : -INFINITY;
#pragma unroll
                for (int r = 1; r < DRBN; ++r) s[i][r] = -INFINITY;
            }
            fold(s, vf, 1);
        }
    }
#pragma unroll
    for (int i = 0; i < NQ; ++i)
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int o = 16; o >= LPK; o >>= 1) acc[i][x] += __shfl_xor_sync(0xffffffffu, acc[i][x], o);
    if (live && grp == 0) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            const float inv = 1.0f / l[i];
            uint4 w;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                __nv_bfloat162 p2 =
                    __floats2bfloat162_rn(acc[i][2 * x] * inv, acc[i][2 * x + 1] * inv);
                wp[x] = *reinterpret_cast<uint32_t*>(&p2);
            }
            *reinterpret_cast<uint4*>(A + (size_t)(b * NQ + i) * d + h * DH + seg * 8) = w;
        }
        if (SWA && W > 1) {
            // every read of this head's ring is done: the block's positions
            // enter slots (pd + e) mod (W-1), the last min(NQ, W-1) of them
#pragma unroll
            for (int e = 0; e < NQ; ++e) {
                if (NQ - e > span) continue;
                const size_t slot = (size_t)((pd + e) % span) * DH;
                *reinterpret_cast<uint4*>(const_cast<bf16*>(kg) + slot) =
                    *reinterpret_cast<const uint4*>(&s_k[warp][e][seg * 8]);
                *reinterpret_cast<uint4*>(const_cast<bf16*>(vg) + slot) =
                    *reinterpret_cast<const uint4*>(&s_v[warp][e][seg * 8]);
            }
        }
    }
}

template <bool SWA>
bool launch_decn64(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W,
                   bf16* A, int B, int n, int heads, const ProjIn& pin, cudaStream_t st) {
    const int grid = (B * heads + DWARPS - 1) / DWARPS;
    if (n == 2)
        launch(k_attn_decn<64, SWA, 2>, grid, DWARPS * 32, 0, st, base, row_stride, span, pos, W,
               A, B, heads, pin);
    else if (n == 3)
        launch(k_attn_decn<64, SWA, 3>, grid, DWARPS * 32, 0, st, base, row_stride, span, pos, W,
               A, B, heads, pin);
    else
        launch(k_attn_decn<64, SWA, 4>, grid, DWARPS * 32, 0, st, base, row_stride, span, pos, W,
               A, B, heads, pin);
    rlt_count_launch();
    return true;
}

// One-position cross-attention with the keys of one (row, head) split over
// the XS warps of a CTA (flash-decoding style): warp w streams the w-th
// contiguous part of keys 1..t exactly as k_attn_dec1 streams a whole run
// (two batches in flight), then the warps' partial maxima, sums and outputs
// are merged in warp order.  Each warp's chain of dependent loads is XS
// times shorter.  The split depends on t and the head size alone, so a row's
// result does not depend on its batch.
// QIN: the query is read ready-rotated from an fp32 [B][d] buffer (pin.P,
// row pitch pin.ldp) -- the encoder's generation steps -- instead of being
// formed from projection slabs.
// SWA: the window attention over the ring's occupied slots 0 .. min(pd, W-1)-1
// (split over the warps the same way), then the position's own key, formed
// from the slabs by warp 0 and folded into its part; after the merge the
// position enters its ring slot (every warp has finished reading the ring).
template <int DH, int XS, bool QIN = false, bool SWA = false>
__global__ void __launch_bounds__(XS * 32)
k_attn_xsplit(const bf16* __restrict__ base, size_t row_stride, int span,
              const int32_t* __restrict__ pos, bf16* __restrict__ A, int heads, ProjIn pin,
              int W) {
    constexpr int LPK = DH / 8, KPR = 32 / LPK, HALF = DH / 2;
    constexpr int BATCH = DRB * KPR;             // keys per batch
    __shared__ __align__(16) float s_q[DH];
    __shared__ float s_m[XS], s_l[XS];
    __shared__ __align__(16) float s_o[XS][DH];
    __shared__ __align__(16) bf16 s_k[SWA ? DH : 8], s_v[SWA ? DH : 8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / heads, h = blockIdx.x % heads;
    const int d = heads * DH, seg = lane % LPK, grp = lane / LPK;
    const int t0 = __ldcg(pos + b) + 1;
    // debug builds: keys 1..t (memory) and the RoPE row of t must exist
    // (else no keys)
    const bool live = dcheck(t0 >= 1 && (SWA || t0 <= span) && t0 <= pin.rope.max_pos,
                             &g_attn_error, kDevCapacity);
    const int t = live ? t0 : 0;
    // the run: memory keys 0..t-1, or the ring's occupied slots
    const int nrun = SWA ? (live && W > 1 ? min(t0 - 1, span) : 0) : t;
    // warp w: keys [jlo, jhi) of the run, parts rounded to whole batches
    const int part = ((nrun + XS - 1) / XS + BATCH - 1) / BATCH * BATCH;
    const int jlo = min(nrun, warp * part), jhi = min(nrun, jlo + part);
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH + seg * 8;
    const bf16* vg = kg + (size_t)heads * span * DH;
    // memory lines stay in L2 for the next blocks; the ring streams
    const uint64_t l2pol = SWA ? 0 : l2_evict_last_policy();
    uint4 kb0[DRB], vb0[DRB], kb1[DRB], vb1[DRB];
    auto load_batch = [&](int j0, uint4 (&kb)[DRB], uint4 (&vb)[DRB]) {
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            const int j = j0 + r * KPR + grp;
            if (j < jhi) {
                kb[r] = ld_kv<!SWA>(kg + (size_t)j * DH, l2pol);
                vb[r] = ld_kv<!SWA>(vg + (size_t)j * DH, l2pol);
            }
        }
    };
    // the memory was written two or more kernels back: its first keys are
    // requested before the wait for the previous kernel; the encoder cache
    // (QIN) holds the new position's key, written by the kernel just before
    if (QIN) pdl_enter();
    if (jlo < jhi) load_batch(jlo, kb0, vb0);
    if (jlo + BATCH < jhi) load_batch(jlo + BATCH, kb1, vb1);
    if (!QIN) pdl_enter();

    // q: formed once by warp 0 (rotate-half pairs at position t, slab sums in
    // slab order), shared by the four warps
    if (QIN) {
        for (int j = threadIdx.x; j < DH; j += XS * 32)
            s_q[j] = pin.P[(size_t)b * pin.ldp + h * DH + j];
    } else if (warp == 0) {
        const size_t rb = (size_t)b * pin.ldp + h * DH;
        const float* cs = pin.rope.cs + (size_t)t * HALF;
        const float* sn = pin.rope.sn + (size_t)t * HALF;
        for (int j = lane; j < HALF; j += 32) {
            float y1, y2;
            rope_pair(slab_sum8(pin.P, pin.S, pin.slab, rb + j),
                     slab_sum8(pin.P, pin.S, pin.slab, rb + j + HALF), cs[j], sn[j], y1, y2);
            s_q[j] = y1;
            s_q[j + HALF] = y2;
        }
    }
    __syncthreads();
    const float sc = 1.0f / sqrtf((float)DH);
    float q[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) q[x] = s_q[seg * 8 + x] * sc;

    float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) acc[x] = 0.f;
    auto fold = [&](int j0, const uint4 (&kb)[DRB], const uint4 (&vb)[DRB]) {
        float s[DRB];
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            const bool v = j0 + r * KPR + grp < jhi;
            float kf[8] = {};
            if (v) unpack8(kb[r], kf);
            float dot = 0.f;
#pragma unroll
            for (int x = 0; x < 8; ++x) dot = fmaf(q[x], kf[x], dot);
#pragma unroll
            for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            s[r] = v ? dot : -INFINITY;
        }
        float bm = s[0];
#pragma unroll
        for (int r = 1; r < DRB; ++r) bm = fmaxf(bm, s[r]);
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        const float mn = fmaxf(m, bm);          // finite: the batch holds a key
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        float ps = 0.f;
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            s[r] = (s[r] == -INFINITY) ? 0.f : __expf(s[r] - mn);
            ps += s[r];
        }
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        l = l * corr + ps;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] *= corr;
        m = mn;
#pragma unroll
        for (int r = 0; r < DRB; ++r) {
            if (!(j0 + r * KPR + grp < jhi)) continue;
            float vf[8];
            unpack8(vb[r], vf);
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = fmaf(s[r], vf[x], acc[x]);
        }
    };
    for (int j0 = jlo; j0 < jhi; j0 += 2 * BATCH) {
        fold(j0, kb0, vb0);
        if (j0 + 2 * BATCH < jhi) load_batch(j0 + 2 * BATCH, kb0, vb0);
        if (j0 + BATCH >= jhi) break;
        fold(j0 + BATCH, kb1, vb1);
        if (j0 + 3 * BATCH < jhi) load_batch(j0 + 3 * BATCH, kb1, vb1);
    }
    if (SWA && warp == 0 && live) {
        // the position's own k and v, rounded like the stored ones; every
        // lane group scores the key, group 0 carries its value
        const size_t rb = (size_t)b * pin.ldp + h * DH;
        const float* cs = pin.rope.cs + (size_t)t * HALF;
        const float* sn = pin.rope.sn + (size_t)t * HALF;
        for (int j = lane; j < HALF; j += 32) {
            float y1, y2;
            rope_pair(slab_sum8(pin.P, pin.S, pin.slab, rb + d + j),
                      slab_sum8(pin.P, pin.S, pin.slab, rb + d + j + HALF), cs[j], sn[j], y1, y2);
            s_k[j] = __float2bfloat16_rn(y1);
            s_k[j + HALF] = __float2bfloat16_rn(y2);
            s_v[j] = __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + j));
            s_v[j + HALF] = __float2bfloat16_rn(slab_sum8(pin.P, pin.S, pin.slab, rb + 2 * d + j + HALF));
        }
        __syncwarp();
        float kf[8], vf[8];
        unpack8(*reinterpret_cast<const uint4*>(&s_k[seg * 8]), kf);
        unpack8(*reinterpret_cast<const uint4*>(&s_v[seg * 8]), vf);
        float dot = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) dot = fmaf(q[x], kf[x], dot);
#pragma unroll
        for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float mn = fmaxf(m, dot);
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        const float p = __expf(dot - mn);
        l = l * corr + p;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] = acc[x] * corr + (grp == 0 ? p * vf[x] : 0.f);
        m = mn;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int o = 16; o >= LPK; o >>= 1) acc[x] += __shfl_xor_sync(0xffffffffu, acc[x], o);
    if (grp == 0) {
#pragma unroll
        for (int x = 0; x < 8; ++x) s_o[warp][seg * 8 + x] = acc[x];
        if (lane == 0) {
            s_m[warp] = m;
            s_l[warp] = l;
        }
    }
    __syncthreads();
    // merge the parts in warp order (part 0 always holds key 1)
    for (int x = threadIdx.x; live && x < DH; x += XS * 32) {
        float M = s_m[0];
#pragma unroll
        for (int w = 1; w < XS; ++w) M = fmaxf(M, s_m[w]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < XS; ++w) {
            if (s_m[w] == -INFINITY) continue;
            const float f = __expf(s_m[w] - M);
            L += s_l[w] * f;
            O += s_o[w][x] * f;
        }
        A[(size_t)b * d + h * DH + x] = __float2bfloat16_rn(O / L);
    }
    if (SWA && live && W > 1) {
        // every warp has read its part of the ring (the barrier above): the
        // position enters slot pd mod (W-1)
        bf16* rk = const_cast<bf16*>(base) + (size_t)b * row_stride + (size_t)h * span * DH +
                   (size_t)((t0 - 1) % span) * DH;
        bf16* rv = rk + (size_t)heads * span * DH;
        for (int x = threadIdx.x; x < DH; x += XS * 32) {
            rk[x] = s_k[x];
            rv[x] = s_v[x];
        }
    }
}

template <int DH, bool SWA>
bool launch_dec1(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W, bf16* A,
                 int B, int heads, const ProjIn& pin, cudaStream_t st) {
    const int items = B * heads;
    launch(k_attn_dec1<DH, SWA>, (items + DWARPS - 1) / DWARPS, DWARPS * 32, 0, st, base,
           row_stride, span, pos, W, A, B, heads, pin);
    rlt_count_launch();
    return true;
}

template <int DH, int NQ, bool SWA, bool PRO, int NSTG>
bool launch_one(const float* Q, const bf16* base, size_t row_stride, int span, const bf16* Kc,
                const bf16* Vc, const int32_t* pos, int W, bf16* A, int B, int n, int heads,
                const ProjIn& pin, cudaStream_t st) {
    constexpr size_t smem = 2 * NSTG * (size_t)CH * DH * 2;
    if (!set_smem_once(reinterpret_cast<const void*>(k_attn_stream<DH, NQ, SWA, PRO, NSTG>), smem))
        return false;
    launch(k_attn_stream<DH, NQ, SWA, PRO, NSTG>, dim3(B * heads, (n + NQ - 1) / NQ), NW * 32,
           smem, st, Q, base, row_stride, span, Kc, Vc, pos, W, A, n, heads, pin);
    rlt_count_launch();
    return true;
}

// One pipeline stage when no run can exceed one chunk (a window of at most
// CH + 1 keys): the smaller footprint keeps twice as many CTAs resident.
template <int DH, bool SWA, bool PRO, int NSTG>
bool launch_stream_n(const float* Q, const bf16* base, size_t row_stride, int span,
                     const bf16* Kc, const bf16* Vc, const int32_t* pos, int W, bf16* A, int B,
                     int n, int heads, const ProjIn& pin, cudaStream_t st) {
    if (n == 1)
        return launch_one<DH, 1, SWA, PRO, NSTG>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B,
                                                 n, heads, pin, st);
    if (n == 2)
        return launch_one<DH, 2, SWA, PRO, NSTG>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B,
                                                 n, heads, pin, st);
    return launch_one<DH, 4, SWA, PRO, NSTG>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B, n,
                                             heads, pin, st);
}

template <int DH, bool SWA, bool PRO>
bool launch_stream(const float* Q, const bf16* base, size_t row_stride, int span, const bf16* Kc,
                   const bf16* Vc, const int32_t* pos, int W, bf16* A, int B, int n, int heads,
                   const ProjIn& pin, cudaStream_t st) {
    // the longest run: the ring's slots, or the whole memory / cache prefix
    if (span <= CH)
        return launch_stream_n<DH, SWA, PRO, 1>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B,
                                                n, heads, pin, st);
    return launch_stream_n<DH, SWA, PRO, 2>(Q, base, row_stride, span, Kc, Vc, pos, W, A, B, n,
                                            heads, pin, st);
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

// Blocks of 2..4 positions (RLT-2 chunks) on one warp per (row, head);
// RLT_DECN=0 keeps them on the shared-memory pipeline kernel (read once).
static bool multi_query_warp() {
    static const bool on = [] {
        const char* e = getenv("RLT_DECN");
        return !(e && strcmp(e, "0") == 0);
    }();
    return on;
}

// RLT_XSPLIT=2 or 4: the one-position cross-attention at d_h = 64 splits
// each (row, head) over that many warps (read once per process).
static int xsplit64() {
    static const int v = [] {
        const char* e = getenv("RLT_XSPLIT");
        const int x = e ? atoi(e) : 0;
        return (x == 2 || x == 4) ? x : 0;
    }();
    return v;
}

bool launch_attn_swa_proj(const ProjIn& pin, bf16* ring, size_t row_stride, int W,
                          const int32_t* pos, bf16* A, int B, int n, int heads, int dh,
                          cudaStream_t st) {
    // one query group per (sequence, head): the kernel then owns every read
    // and write of that head's ring for the block
    if (!fast_attn_enabled() || (dh != 64 && dh != 128)) return false;
    if (B * n <= 0) return true;
    const int slots = W > 1 ? W - 1 : 1;
    if (n >= 2 && W > n &&
        launch_attn_mq<true>(ring, row_stride, slots, pos, W, A, B, n, heads, dh, pin, st))
        return true;
    if (n > 4) return false;
    static const bool xswa = [] {      // RLT_XSPLIT_SWA=0: one warp per item (read once)
        const char* e = getenv("RLT_XSPLIT_SWA");
        return !(e && strcmp(e, "0") == 0);
    }();
    if (n == 1 && pin.S <= 8 && dh == 128 && xswa) {
        // the wide heads' long windows with few items per launch: split each
        // item's ring over four warps
        launch(k_attn_xsplit<128, 4, false, true>, B * heads, 4 * 32, 0, st, ring, row_stride,
               slots, pos, A, heads, pin, W);
        rlt_count_launch();
        return true;
    }
    if (n == 1 && launch_attn_sq<true>(ring, row_stride, slots, pos, W, A, B, heads, dh, pin, st))
        return true;
    if (n == 1 && pin.S <= 8)
        return dh == 64 ? launch_dec1<64, true>(ring, row_stride, slots, pos, W, A, B, heads, pin, st)
                        : launch_dec1<128, true>(ring, row_stride, slots, pos, W, A, B, heads, pin, st);
    if (dh == 64 && pin.S <= 8 && W > 4 && multi_query_warp())
        return launch_decn64<true>(ring, row_stride, slots, pos, W, A, B, n, heads, pin, st);
    if (dh == 64)
        return launch_stream<64, true, true>(nullptr, ring, row_stride, slots, nullptr, nullptr,
                                             pos, W, A, B, n, heads, pin, st);
    return launch_stream<128, true, true>(nullptr, ring, row_stride, slots, nullptr, nullptr, pos,
                                          W, A, B, n, heads, pin, st);
}

bool launch_attn_enc_step(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
                          const int32_t* pos_enc, bf16* A, int B, int heads, int dh,
                          cudaStream_t st) {
    // one new position per row over a long cache prefix, d_h = 128: the
    // split-key kernel, the query already rotated in Q (RLT_ENC_STEP=stream
    // keeps these on the shared-memory pipeline kernel; read once)
    static const bool on = [] {
        const char* e = getenv("RLT_ENC_STEP");
        return !(e && strcmp(e, "stream") == 0);
    }();
    if (!on || !fast_attn_enabled() || dh != 128) return false;
    if (B <= 0) return true;
    ProjIn pin{};
    pin.P = Q;
    pin.S = 1;
    pin.ldp = heads * dh;
    pin.rope.max_pos = T_cap;
    launch(k_attn_xsplit<128, 4, true>, B * heads, 4 * 32, 0, st, cache, row_stride, T_cap,
           pos_enc, A, heads, pin, 0);
    rlt_count_launch();
    return true;
}

bool launch_attn_cross_proj(const ProjIn& pin, const bf16* mem, size_t row_stride, int T_cap,
                            const int32_t* pos, bf16* A, int B, int n, int heads, int dh,
                            cudaStream_t st) {
    if (!fast_attn_enabled() || (dh != 64 && dh != 128)) return false;
    if (B * n <= 0) return true;
    if (n == 1 && pin.S <= 8 && dh == 128) {
        // the wide heads come with long memory prefixes and few items per
        // launch: split each item's keys over four warps
        launch(k_attn_xsplit<128, 4>, B * heads, 4 * 32, 0, st, mem, row_stride, T_cap, pos, A,
               heads, pin, 0);
        rlt_count_launch();
        return true;
    }
    if (n == 1 && pin.S <= 8 && dh == 64 && xsplit64() > 1) {
        if (xsplit64() == 2)
            launch(k_attn_xsplit<64, 2>, B * heads, 2 * 32, 0, st, mem, row_stride, T_cap, pos,
                   A, heads, pin, 0);
        else
            launch(k_attn_xsplit<64, 4>, B * heads, 4 * 32, 0, st, mem, row_stride, T_cap, pos,
                   A, heads, pin, 0);
        rlt_count_launch();
        return true;
    }
    if (n == 1 && launch_attn_sq<false>(mem, row_stride, T_cap, pos, 0, A, B, heads, dh, pin, st))
        return true;
    if (n == 1 && pin.S <= 8)
        return dh == 64 ? launch_dec1<64, false>(mem, row_stride, T_cap, pos, 0, A, B, heads, pin, st)
                        : launch_dec1<128, false>(mem, row_stride, T_cap, pos, 0, A, B, heads, pin, st);
    if (n >= 2 && launch_attn_mq<false>(mem, row_stride, T_cap, pos, 0, A, B, n, heads, dh, pin, st))
        return true;
    if (dh == 64 && pin.S <= 8 && n <= 4 && multi_query_warp())
        return launch_decn64<false>(mem, row_stride, T_cap, pos, 0, A, B, n, heads, pin, st);
    if (dh == 64)
        return launch_stream<64, false, true>(nullptr, mem, row_stride, T_cap, nullptr, nullptr,
                                              pos, 0, A, B, n, heads, pin, st);
    return launch_stream<128, false, true>(nullptr, mem, row_stride, T_cap, nullptr, nullptr, pos,
                                           0, A, B, n, heads, pin, st);
}

}  // namespace rlt
