// One position per row (n = 1, the decode shape) at d_h = 64: the window
// self-attention over the ring cache C^D plus the position itself, and the
// cross-attention over the memory prefix M_{<=t} (jiphyeonjeon review
// "Recurrent Looped Transformer" §2-§3.3; greeksharifa §2.5), on the CUDA
// cores -- a one-position block is a matrix-vector product per (row, head).
#include <math.h>

#include <cstdlib>
#include <cstring>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

constexpr int SQ_TILE = 16;                  // keys per tile
constexpr int SQ_TB = SQ_TILE * 64 * 2;      // bytes of one 16 x 64 bf16 tile

__device__ int g_sq_error;   // sticky: a bounded wait gave up, or a debug-build check failed

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// sum of S (<= 8) split-K partial slabs at element i, in slab order
__device__ __forceinline__ float slab_sum(const float* __restrict__ P, int S, size_t slab,
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

// One position per row (n = 1, the decode shape) at d_h = 64, on the CUDA
// cores: one warp per (row, head).  The keys of a (row, head) are one
// contiguous run per K and V, so a 16-key tile is one 2 KB bulk copy of each
// (lane 0 issues them, completion counted on a per-stage mbarrier, three
// tiles in flight): the bytes in flight hold no registers and issuing a tile
// costs two instructions.  Scores: two lanes per key, 32 dims each, read in
// a per-key rotated chunk order (so that the 8 lanes of a shared-memory
// phase hit 8 different banks groups without a swizzle), packed fp32x2
// FMAs, one shuffle; an online softmax per tile (one warp maximum); values:
// lane group g takes keys 4i+g, 8 dims per lane, packed FMAs, the groups'
// partial outputs added at the end.  q and p stay fp32.  The window form
// folds the position's own key (formed from the slabs) after the ring's
// tiles and then writes it into the ring.  Waits are bounded: a wait that
// gives up records a timeout, the warp stops, and it waits (bounded) for the
// copies it has in flight before it exits.
constexpr int SQ_WARPS = 4;
// NST tiles in flight per warp; per warp NST (K, V) tile pairs, q (fp32)
// and the own k and v
constexpr int sq_warp_smem(int nst) { return nst * 2 * SQ_TB + 512; }
constexpr int sq_smem(int nst) { return SQ_WARPS * sq_warp_smem(nst); }

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
        : "memory");
}
// d = a * b + c on a pair of fp32 values (one packed instruction)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    unsigned long long ua, ub, uc, ud;
    memcpy(&ua, &a, 8);
    memcpy(&ub, &b, 8);
    memcpy(&uc, &c, 8);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ud) : "l"(ua), "l"(ub), "l"(uc));
    float2 d;
    memcpy(&d, &ud, 8);
    return d;
}

template <bool SWA, int SQ_NST>
__global__ void __launch_bounds__(SQ_WARPS * 32)
k_attn_sq(const bf16* __restrict__ base, size_t row_stride, int span,
          const int32_t* __restrict__ pos, int W, bf16* __restrict__ A, int B, int heads,
          ProjIn pin) {
    constexpr int DH = 64, HALF = 32;
    extern __shared__ __align__(1024) uint8_t sq_smem_raw[];
    __shared__ uint64_t bars[SQ_WARPS][SQ_NST];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int it = blockIdx.x * SQ_WARPS + warp;
    const bool in_range = it < B * heads;
    const int b = in_range ? it / heads : 0, h = in_range ? it % heads : 0;
    const int d = heads * DH;
    const int pd = in_range ? __ldcg(pos + b) : 0, t = pd + 1;
    const bool live = in_range && dcheck(pd >= 0 && t <= pin.rope.max_pos && (SWA || t <= span),
                                         &g_sq_error, kDevCapacity);
    // the run: ring slots 0 .. min(pd, W-1)-1, or memory keys 1 .. t
    const int nrun = !live ? 0 : (SWA ? (W > 1 ? min(pd, span) : 0) : t);
    const int ntile = (nrun + SQ_TILE - 1) / SQ_TILE;
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH;
    const bf16* vg = kg + (size_t)heads * span * DH;
    uint8_t* wsm = sq_smem_raw + warp * sq_warp_smem(SQ_NST);
    const uint32_t sKV = tc::smem_u32(wsm);
    float* s_q = reinterpret_cast<float*>(wsm + SQ_NST * 2 * SQ_TB);    // 64 floats
    bf16* s_k = reinterpret_cast<bf16*>(s_q + DH);                      // own k, v
    bf16* s_v = s_k + DH;
    uint64_t* bar = bars[warp];
    if (lane == 0) {
        for (int s = 0; s < SQ_NST; ++s) tc::mbar_init(&bar[s], 1);
        tc::fence_mbar_init();
    }
    __syncwarp();

    // tile k of the run (its first min(16, nrun - 16k) keys) into stage k % NST
    auto issue = [&](int k) {
        if (lane == 0 && k < ntile) {
            const int s = k % SQ_NST, nv = min(SQ_TILE, nrun - k * SQ_TILE);
            const uint32_t bytes = (uint32_t)nv * DH * 2;
            tc::mbar_expect_tx(&bar[s], 2 * bytes);
            const uint32_t stK = sKV + (uint32_t)(2 * s) * SQ_TB;
            bulk_copy(stK, kg + (size_t)k * SQ_TILE * DH, bytes, &bar[s]);
            bulk_copy(stK + SQ_TB, vg + (size_t)k * SQ_TILE * DH, bytes, &bar[s]);
        }
    };
    // ring and memory were written two or more kernels back
#pragma unroll
    for (int k = 0; k < SQ_NST; ++k) issue(k);
    pdl_enter();

    // q (rotated, scaled) and, for the window, the position's own k and v
    const float sc = 0.125f;                         // 1 / sqrt(64)
    if (live) {
        const size_t rb = (size_t)b * pin.ldp + h * DH;
        const float* cs = pin.rope.cs + (size_t)t * HALF;
        const float* sn = pin.rope.sn + (size_t)t * HALF;
        const int j = lane;
        float y1, y2;
        rope_pair(slab_sum(pin.P, pin.S, pin.slab, rb + j),
                  slab_sum(pin.P, pin.S, pin.slab, rb + j + HALF), cs[j], sn[j], y1, y2);
        s_q[j] = y1 * sc;
        s_q[j + HALF] = y2 * sc;
        if (SWA) {
            rope_pair(slab_sum(pin.P, pin.S, pin.slab, rb + d + j),
                      slab_sum(pin.P, pin.S, pin.slab, rb + d + j + HALF), cs[j], sn[j], y1, y2);
            s_k[j] = __float2bfloat16_rn(y1);
            s_k[j + HALF] = __float2bfloat16_rn(y2);
            s_v[j] = __float2bfloat16_rn(slab_sum(pin.P, pin.S, pin.slab, rb + 2 * d + j));
            s_v[j + HALF] = __float2bfloat16_rn(slab_sum(pin.P, pin.S, pin.slab, rb + 2 * d + j + HALF));
        }
    }
    __syncwarp();
    // scores: lane 2r+hf takes dims 32hf .. 32hf+31 of key r of a tile, in
    // the chunk order 4hf + (u + r) mod 4, u = 0..3; its q in that order
    const int kr = lane >> 1, hf = lane & 1;
    float2 q2[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const float* src = s_q + 32 * hf + 8 * ((u + kr) & 3);
#pragma unroll
        for (int x = 0; x < 4; ++x) q2[4 * u + x] = make_float2(src[2 * x], src[2 * x + 1]);
    }
    // values: lane group g (lane / 8) takes keys 4i+g, dims 8*seg .. 8*seg+7
    const int grp = lane >> 3, seg = lane & 7;
    float m = -INFINITY, lpart = 0.f;
    float2 acc[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[x] = make_float2(0.f, 0.f);
    int kfail = -1;                                  // tile whose copy never completed

    for (int k = 0; k < ntile; ++k) {
        const int s = k % SQ_NST;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&bar[s], (uint32_t)(k / SQ_NST) & 1u))) {
            kfail = k;
            break;
        }
        const int nv = min(SQ_TILE, nrun - k * SQ_TILE);
        const uint8_t* tK = wsm + 2 * s * SQ_TB;
        const uint8_t* tV = tK + SQ_TB;
        float2 dd = make_float2(0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint4 w = *reinterpret_cast<const uint4*>(tK + kr * 128 +
                                                            (4 * hf + ((u + kr) & 3)) * 16);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
            for (int x = 0; x < 4; ++x) dd = fma2(q2[4 * u + x], __bfloat1622float2(h2[x]), dd);
        }
        float dot = dd.x + dd.y;
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        const bool vis = kr < nv;
        const float sv = vis ? dot : -INFINITY;
        float tm = sv;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, o));
        const float mn = fmaxf(m, tm);               // finite: the tile holds a key
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        const float p = vis ? __expf(sv - mn) : 0.f;
        lpart = lpart * corr + (hf == 0 ? p : 0.f);
        m = mn;
        const float2 c2 = make_float2(corr, corr);
#pragma unroll
        for (int x = 0; x < 4; ++x) acc[x] = make_float2(acc[x].x * c2.x, acc[x].y * c2.y);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * i + grp;
            const float pj = __shfl_sync(0xffffffffu, p, 2 * j);
            if (j < nv) {                            // rows past the copy hold stale bytes
                const uint4 w = *reinterpret_cast<const uint4*>(tV + j * 128 + seg * 16);
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
                const float2 p2 = make_float2(pj, pj);
#pragma unroll
                for (int x = 0; x < 4; ++x) acc[x] = fma2(p2, __bfloat1622float2(h2[x]), acc[x]);
            }
        }
        __syncwarp();                                // the stage is read: refill it
        issue(k + SQ_NST);
    }
    if (kfail >= 0) {
        // a copy never completed: record it, then wait (bounded) for the
        // copies still in flight -- tiles kfail .. kfail+NST-1 were issued --
        // so that none lands after the warp is gone
        if (lane == 0) {
            atomicExch(&g_sq_error, kDevTimeout);
            for (int k = kfail; k < min(ntile, kfail + SQ_NST); ++k)
                tc::mbar_wait(&bar[k % SQ_NST], (uint32_t)(k / SQ_NST) & 1u, 1u << 20);
        }
        return;
    }
    if (SWA && live) {
        // the position itself: every lane pair scores it, lane 0 counts it,
        // group 0 carries its value
        float2 dd = make_float2(0.f, 0.f);
#pragma unroll
        for (int x = 0; x < 16; ++x) {
            const float2 kf = __bfloat1622float2(
                *reinterpret_cast<const __nv_bfloat162*>(s_k + 32 * hf + 2 * x));
            dd = fma2(make_float2(s_q[32 * hf + 2 * x], s_q[32 * hf + 2 * x + 1]), kf, dd);
        }
        float dot = dd.x + dd.y;
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        const float mn = fmaxf(m, dot);
        const float corr = (m == -INFINITY) ? 0.f : __expf(m - mn);
        const float p = __expf(dot - mn);
        lpart = lpart * corr + (lane == 0 ? p : 0.f);
        m = mn;
        const uint4 w = *reinterpret_cast<const uint4*>(s_v + 8 * seg);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float2 vf = __bfloat1622float2(h2[x]);
            acc[x].x = acc[x].x * corr + (grp == 0 ? p * vf.x : 0.f);
            acc[x].y = acc[x].y * corr + (grp == 0 ? p * vf.y : 0.f);
        }
    }
    // the normaliser and the output: sums over the lanes and over the groups
    float l = lpart;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        acc[x].x += __shfl_xor_sync(0xffffffffu, acc[x].x, 8);
        acc[x].y += __shfl_xor_sync(0xffffffffu, acc[x].y, 8);
        acc[x].x += __shfl_xor_sync(0xffffffffu, acc[x].x, 16);
        acc[x].y += __shfl_xor_sync(0xffffffffu, acc[x].y, 16);
    }
    if (live && grp == 0) {
        const float inv = 1.0f / l;
        uint4 w;
        w.x = pack_bf16(acc[0].x * inv, acc[0].y * inv);
        w.y = pack_bf16(acc[1].x * inv, acc[1].y * inv);
        w.z = pack_bf16(acc[2].x * inv, acc[2].y * inv);
        w.w = pack_bf16(acc[3].x * inv, acc[3].y * inv);
        *reinterpret_cast<uint4*>(A + (size_t)b * d + h * DH + 8 * seg) = w;
        if (SWA && W > 1) {
            // every read of this head's ring is done: the position enters
            // slot pd mod (W-1)
            const size_t slot = (size_t)(pd % span) * DH + 8 * seg;
            *reinterpret_cast<uint4*>(const_cast<bf16*>(kg) + slot) =
                *reinterpret_cast<const uint4*>(s_k + 8 * seg);
            *reinterpret_cast<uint4*>(const_cast<bf16*>(vg) + slot) =
                *reinterpret_cast<const uint4*>(s_v + 8 * seg);
        }
    }
}

}  // namespace

int read_and_clear_sq_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_sq_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        int z = 0;
        cudaMemcpyToSymbol(g_sq_error, &z, sizeof(int));
    }
    return v;
}

// RLT_SQ=0 keeps one-position blocks on the register-batch kernel (read once).
static bool sq_enabled() {
    static const bool on = [] {
        const char* e = getenv("RLT_SQ");
        return !(e && e[0] == '0' && e[1] == 0);
    }();
    return on;
}

// Key tiles in flight per warp: two for the window (at most four tiles of
// ring, the first two requested before the previous kernel ends), three for
// the memory prefix (measured best on the parity and S5 workloads; four
// leave fewer warps resident than one wave needs).  RLT_SQ_STAGES=2|3|4
// sets both (read once).
static int sq_stages(bool swa) {
    static const int v = [] {
        const char* e = getenv("RLT_SQ_STAGES");
        const int n = e ? atoi(e) : 0;
        return (n >= 2 && n <= 4) ? n : 0;
    }();
    return v ? v : (swa ? 2 : 3);
}

template <bool SWA, int NST>
bool launch_sq_nst(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W,
                   bf16* A, int B, int heads, const ProjIn& pin, cudaStream_t st) {
    if (!set_smem_once(reinterpret_cast<const void*>(k_attn_sq<SWA, NST>), sq_smem(NST)))
        return false;
    launch(k_attn_sq<SWA, NST>, (B * heads + SQ_WARPS - 1) / SQ_WARPS, SQ_WARPS * 32,
           sq_smem(NST), st, base, row_stride, span, pos, W, A, B, heads, pin);
    rlt_count_launch();
    return true;
}

template <bool SWA>
bool launch_attn_sq(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W,
                    bf16* A, int B, int heads, int dh, const ProjIn& pin, cudaStream_t st) {
    if (!sq_enabled() || dh != 64 || pin.S > 8) return false;
    if (B <= 0) return true;
    switch (sq_stages(SWA)) {
        case 2: return launch_sq_nst<SWA, 2>(base, row_stride, span, pos, W, A, B, heads, pin, st);
        case 4: return launch_sq_nst<SWA, 4>(base, row_stride, span, pos, W, A, B, heads, pin, st);
        default: return launch_sq_nst<SWA, 3>(base, row_stride, span, pos, W, A, B, heads, pin, st);
    }
}
template bool launch_attn_sq<true>(const bf16*, size_t, int, const int32_t*, int, bf16*, int, int,
                                   int, const ProjIn&, cudaStream_t);
template bool launch_attn_sq<false>(const bf16*, size_t, int, const int32_t*, int, bf16*, int,
                                    int, int, const ProjIn&, cudaStream_t);

}  // namespace rlt
