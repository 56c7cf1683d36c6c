// Decoder attention for blocks of NQ = 2..16 positions per row (RLT-2 chunks,
// RLT-0 blocks) at d_h = 64: the window self-attention over the ring
// cache C^D plus the block's own positions, and the cross-attention over the
// memory prefix M_{<=t} (jiphyeonjeon review "Recurrent Looped Transformer"
// §2-§3.3; greeksharifa §2.5, §2.7 and App. I.2 for the blocks).
//
// Every key of a (row, head) serves the NQ queries of the block, so the
// scores of a 16-key tile are the product Q (NQ x 64) . K^T and the output a
// product P . V: one warp per (row, head) runs both on the warp-level tensor
// core MMA (m16n8k16, bf16 operands, fp32 accumulation; the NQ queries fill
// rows 0..NQ-1 of the 16-row operand, each lane carrying the softmax of rows
// lane/4 and, past 8 queries, lane/4 + 8).  The work stays an HBM stream -- each
// key and value is read once -- and the products only cut the per-key
// instruction count that bounds the CUDA-core form of the same loop.
//
// Keys and values reach shared memory by cp.async, 16-key tiles, three
// tiles in flight per warp, rows XOR-swizzled in 16-byte chunks so that the
// ldmatrix reads are conflict-free.  q and the probabilities enter the
// products as bf16; the softmax normaliser is the sum of the rounded
// probabilities, the same reading as the encoder's tensor-core attention.
// Query i of the block sits at t_i = pd+1+i: the window shows it positions
// max(1, t_i-W+1) .. t_i (ring slots, then the block's own positions e <= i,
// formed from the projection slabs after the ring's tiles are issued); the
// memory shows it positions 1 .. t_i.  After its last read of the ring the
// warp moves the block's positions into their slots.  Key order and every
// reduction order depend on positions only, never on the batch.
#include <math.h>

#include <cstdlib>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

constexpr int MQ_WARPS = 4;                 // (row, head) items per CTA
constexpr int MQ_NST = 3;                   // key tiles in flight per warp
constexpr int MQ_TILE = 16;                 // keys per tile
constexpr int MQ_TB = MQ_TILE * 64 * 2;     // bytes of one 16 x 64 bf16 tile
// per warp: Q tile, NST stages of (K, V) tiles, the block's own (K, V) tile
constexpr int MQ_WARP_SMEM = MQ_TB + MQ_NST * 2 * MQ_TB + 2 * MQ_TB;
constexpr int MQ_SMEM = MQ_WARPS * MQ_WARP_SMEM;

// byte offset of 16-byte chunk c of row r in a [16][64] bf16 tile
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
    // an invalid chunk is zero-filled (no bytes read)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// d += a . b (16 x 8 x 16, bf16 in, fp32 accumulate)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

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


__device__ int g_mq_error;   // sticky: a debug-build bounds check failed

template <bool SWA, int NQ>
__global__ void __launch_bounds__(MQ_WARPS * 32)
k_attn_mq(const bf16* __restrict__ base, size_t row_stride, int span,
          const int32_t* __restrict__ pos, int W, bf16* __restrict__ A, int B, int heads,
          ProjIn pin) {
    constexpr int DH = 64, HALF = 32;
    extern __shared__ __align__(1024) uint8_t mq_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int it = blockIdx.x * MQ_WARPS + warp;
    const bool in_range = it < B * heads;
    const int b = in_range ? it / heads : 0, h = in_range ? it % heads : 0;
    const int d = heads * DH;
    const int pd = in_range ? __ldcg(pos + b) : 0;
    // debug builds: the block's positions must have RoPE rows and (memory)
    // keys inside the buffer; a failed check skips the item
    const bool live = in_range && dcheck(pd >= 0 && pd + NQ <= pin.rope.max_pos &&
                                             (SWA || pd + NQ <= span),
                                         &g_mq_error, kDevCapacity);
    // the run of stored keys: ring slots 0 .. nmain-1, or memory keys 1 .. pd+NQ
    const int nmain = !live ? 0 : (SWA ? (W > 1 ? min(pd, span) : 0) : pd + NQ);
    const int ntile = (nmain + MQ_TILE - 1) / MQ_TILE;
    const bf16* kg = base + (size_t)b * row_stride + (size_t)h * span * DH;
    const bf16* vg = kg + (size_t)heads * span * DH;

    uint8_t* wsm = mq_smem + warp * MQ_WARP_SMEM;
    const uint32_t sQ = tc::smem_u32(wsm);
    const uint32_t sKV = sQ + MQ_TB;                     // stage s: K at +2s*TB, V at +(2s+1)*TB
    const uint32_t sOwnK = sKV + 2 * MQ_NST * MQ_TB, sOwnV = sOwnK + MQ_TB;

    // tile k of the run into stage k % NST: lane copies chunks lane + 32u
    // (row = chunk / 8) of K and of V; keys past the run are zero-filled
    auto issue = [&](int k) {
        if (k < ntile) {
            const uint32_t stK = sKV + (uint32_t)(2 * (k % MQ_NST)) * MQ_TB, stV = stK + MQ_TB;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int ch = lane + 32 * u, r = ch >> 3, c = ch & 7, j = k * MQ_TILE + r;
                const bool ok = j < nmain;
                const size_t off = (size_t)(ok ? j : 0) * DH + c * 8;
                cp16(stK + swz(r, c), kg + off, ok);
                cp16(stV + swz(r, c), vg + off, ok);
            }
        }
        cp_commit();
    };
    // stored keys were written two or more kernels back: request them first
#pragma unroll
    for (int k = 0; k < MQ_NST; ++k) issue(k);
    pdl_enter();

    // the block's queries (bf16, unscaled) in rows 0..NQ-1 of the Q tile,
    // zero rows after; for the window, its own keys and values likewise
    for (int ch = lane; ch < 16 * 8; ch += 32) {
        const int r = ch >> 3, c = ch & 7;
        if (r >= NQ || !live) {
            *reinterpret_cast<uint4*>(wsm + swz(r, c)) = make_uint4(0, 0, 0, 0);
            if (SWA) {
                *reinterpret_cast<uint4*>(wsm + (sOwnK - sQ) + swz(r, c)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(wsm + (sOwnV - sQ) + swz(r, c)) = make_uint4(0, 0, 0, 0);
            }
        }
    }
    if (live) {
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            const size_t rb = (size_t)(b * NQ + i) * pin.ldp + h * DH;
            const float* cs = pin.rope.cs + (size_t)(pd + 1 + i) * HALF;
            const float* sn = pin.rope.sn + (size_t)(pd + 1 + i) * HALF;
            const int j = lane;                      // pair (j, j + 32)
            float y1, y2;
            rope_pair(slab_sum(pin.P, pin.S, pin.slab, rb + j),
                      slab_sum(pin.P, pin.S, pin.slab, rb + j + HALF), cs[j], sn[j], y1, y2);
            bf16* qrow = reinterpret_cast<bf16*>(wsm);
            qrow[(swz(i, j >> 3) >> 1) + (j & 7)] = __float2bfloat16_rn(y1);
            qrow[(swz(i, (j + HALF) >> 3) >> 1) + (j & 7)] = __float2bfloat16_rn(y2);
            if (SWA) {
                rope_pair(slab_sum(pin.P, pin.S, pin.slab, rb + d + j),
                          slab_sum(pin.P, pin.S, pin.slab, rb + d + j + HALF), cs[j], sn[j], y1,
                          y2);
                bf16* krow = reinterpret_cast<bf16*>(wsm + (sOwnK - sQ));
                bf16* vrow = reinterpret_cast<bf16*>(wsm + (sOwnV - sQ));
                krow[(swz(i, j >> 3) >> 1) + (j & 7)] = __float2bfloat16_rn(y1);
                krow[(swz(i, (j + HALF) >> 3) >> 1) + (j & 7)] = __float2bfloat16_rn(y2);
                vrow[(swz(i, j >> 3) >> 1) + (j & 7)] =
                    __float2bfloat16_rn(slab_sum(pin.P, pin.S, pin.slab, rb + 2 * d + j));
                vrow[(swz(i, (j + HALF) >> 3) >> 1) + (j & 7)] =
                    __float2bfloat16_rn(slab_sum(pin.P, pin.S, pin.slab, rb + 2 * d + j + HALF));
            }
        }
    }
    __syncwarp();

    // fragments: lane's 8x8 matrix mi = lane/8, its row lane%8
    const int mi = lane >> 3, r8 = lane & 7;
    uint32_t qa[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
        ldsm4(sQ + swz(r8 + ((mi & 1) << 3), 2 * ks + (mi >> 1)), qa[ks]);

    // this lane's accumulator rows (queries qi and, for blocks of more than
    // 8 positions, qi + 8) and columns
    constexpr int NR = NQ > 8 ? 2 : 1;
    const int qi = lane >> 2, c2 = (lane & 3) * 2;
    bool qrow[NR];
    int t_i[NR], lo[NR];
    float m[NR], lpart[NR];
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) {
        qrow[hh] = live && qi + 8 * hh < NQ;
        t_i[hh] = pd + 1 + qi + 8 * hh;
        lo[hh] = SWA ? max(1, t_i[hh] - W + 1) : 1;    // first visible position
        m[hh] = -INFINITY;
        lpart[hh] = 0.f;
    }
    float o[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int x = 0; x < 4; ++x) o[nt][x] = 0.f;
    const float sc = 0.125f;                         // 1 / sqrt(64)

    // one 16-key tile: kidx0 the run index of its first key (own tile: -1)
    auto fold_tile = [&](uint32_t tK, uint32_t tV, int kidx0) {
        float s[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int x = 0; x < 4; ++x) s[j][x] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t kb[4];
            ldsm4(tK + swz(r8 + ((mi >> 1) << 3), 2 * ks + (mi & 1)), kb);
            mma16816(s[0], qa[ks], kb[0], kb[1]);
            mma16816(s[1], qa[ks], kb[2], kb[3]);
        }
        // row hh of this lane: scores s[j][2hh], s[j][2hh+1] for keys 8j+c2, 8j+c2+1
        float p[NR][4], corr[NR];
#pragma unroll
        for (int hh = 0; hh < NR; ++hh) {
            const int qrw = qi + 8 * hh;
            float v[4];
            bool vis[4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int kt = 8 * j + c2 + x;       // key within the tile
                    bool ok = qrow[hh];
                    if (kidx0 < 0) {                     // own position e = kt
                        ok = ok && kt < NQ && kt <= qrw && pd + 1 + kt >= lo[hh];
                    } else {
                        const int kk = kidx0 + kt;
                        if (SWA) {
                            const int ps = pd - ((pd - 1 - kk) % span);
                            ok = ok && kk < nmain && ps >= lo[hh];
                        } else {
                            ok = ok && kk < nmain && kk + 1 <= t_i[hh];
                        }
                    }
                    vis[2 * j + x] = ok;
                    v[2 * j + x] = s[j][2 * hh + x] * sc;
                }
            float tm = -INFINITY;
#pragma unroll
            for (int x = 0; x < 4; ++x)
                if (vis[x]) tm = fmaxf(tm, v[x]);
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 1));
            tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, 2));
            const float mn = fmaxf(m[hh], tm);
            corr[hh] = 1.f;
#pragma unroll
            for (int x = 0; x < 4; ++x) p[hh][x] = 0.f;
            if (mn != -INFINITY) {
                corr[hh] = (m[hh] == -INFINITY) ? 0.f : __expf(m[hh] - mn);
#pragma unroll
                for (int x = 0; x < 4; ++x) p[hh][x] = vis[x] ? __expf(v[x] - mn) : 0.f;
                m[hh] = mn;
            }
        }
        // P as the A operand: rows qi (and qi + 8), keys c2.. and 8+c2..
        uint32_t pa[4];
        pa[0] = pack_bf16(p[0][0], p[0][1]);
        pa[2] = pack_bf16(p[0][2], p[0][3]);
        if constexpr (NR == 2) {
            pa[1] = pack_bf16(p[NR - 1][0], p[NR - 1][1]);
            pa[3] = pack_bf16(p[NR - 1][2], p[NR - 1][3]);
        } else {
            pa[1] = 0u;
            pa[3] = 0u;
        }
#pragma unroll
        for (int hh = 0; hh < NR; ++hh) {
            // the normaliser sums the rounded probabilities
            const float2 r01 =
                __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pa[hh]));
            const float2 r23 =
                __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&pa[2 + hh]));
            lpart[hh] = lpart[hh] * corr[hh] + ((r01.x + r01.y) + (r23.x + r23.y));
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                o[nt][2 * hh] *= corr[hh];
                o[nt][2 * hh + 1] *= corr[hh];
            }
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t vb[4];
            ldsm4t(tV + swz(r8 + ((mi & 1) << 3), 2 * np + (mi >> 1)), vb);
            mma16816(o[2 * np], pa, vb[0], vb[1]);
            mma16816(o[2 * np + 1], pa, vb[2], vb[3]);
        }
    };

    for (int k = 0; k < ntile; ++k) {
        cp_wait<MQ_NST - 1>();
        __syncwarp();
        const uint32_t stK = sKV + (uint32_t)(2 * (k % MQ_NST)) * MQ_TB;
        fold_tile(stK, stK + MQ_TB, k * MQ_TILE);
        __syncwarp();                                // the stage is read: refill it
        issue(k + MQ_NST);
    }
    cp_wait<0>();
    __syncwarp();
    if (SWA) fold_tile(sOwnK, sOwnV, -1);

    // normaliser: the four lanes of the row hold parts of the sum
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) {
        float l = lpart[hh];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (qrow[hh]) {
            const float inv = 1.0f / l;
            bf16* arow = A + (size_t)(b * NQ + qi + 8 * hh) * d + h * DH + c2;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                *reinterpret_cast<uint32_t*>(arow + nt * 8) =
                    pack_bf16(o[nt][2 * hh] * inv, o[nt][2 * hh + 1] * inv);
        }
    }
    if (SWA && live && W > 1) {
        // every read of this head's ring is done: the block's positions enter
        // slots (pd + e) mod (W-1), the last min(NQ, W-1) of them
        bf16* rk = const_cast<bf16*>(kg);
        bf16* rv = const_cast<bf16*>(vg);
        for (int ch = lane; ch < NQ * 8; ch += 32) {
            const int e = ch >> 3, c = ch & 7;
            if (NQ - e > span) continue;
            const size_t slot = (size_t)((pd + e) % span) * DH + c * 8;
            *reinterpret_cast<uint4*>(rk + slot) =
                *reinterpret_cast<const uint4*>(wsm + (sOwnK - sQ) + swz(e, c));
            *reinterpret_cast<uint4*>(rv + slot) =
                *reinterpret_cast<const uint4*>(wsm + (sOwnV - sQ) + swz(e, c));
        }
    }
}

template <bool SWA, int NQ>
void launch_nq(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W, bf16* A,
               int B, int heads, const ProjIn& pin, cudaStream_t st) {
    launch(k_attn_mq<SWA, NQ>, (B * heads + MQ_WARPS - 1) / MQ_WARPS, MQ_WARPS * 32, MQ_SMEM, st,
           base, row_stride, span, pos, W, A, B, heads, pin);
}

template <bool SWA, int NQ>
bool smem_ok() {
    return set_smem_once(reinterpret_cast<const void*>(k_attn_mq<SWA, NQ>), MQ_SMEM);
}

}  // namespace

int read_and_clear_mq_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_mq_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        int z = 0;
        cudaMemcpyToSymbol(g_mq_error, &z, sizeof(int));
    }
    return v;
}

// RLT_MQ=0 keeps blocks of 2..16 positions on the earlier kernels (read once).
static bool mq_enabled() {
    static const bool on = [] {
        const char* e = getenv("RLT_MQ");
        return !(e && e[0] == '0' && e[1] == 0);
    }();
    return on;
}

template <bool SWA>
bool launch_attn_mq(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W,
                    bf16* A, int B, int n, int heads, int dh, const ProjIn& pin, cudaStream_t st) {
    if (!mq_enabled() || dh != 64 || n < 2 || n > 16 || pin.S > 8) return false;
    if (B * n <= 0) return true;
    bool ok = false;
    switch (n) {
#define RLT_MQ_CASE(N)                                                                     \
    case N:                                                                                \
        ok = smem_ok<SWA, N>();                                                            \
        if (ok) launch_nq<SWA, N>(base, row_stride, span, pos, W, A, B, heads, pin, st); \
        break;
        RLT_MQ_CASE(2)
        RLT_MQ_CASE(3)
        RLT_MQ_CASE(4)
        RLT_MQ_CASE(5)
        RLT_MQ_CASE(6)
        RLT_MQ_CASE(7)
        RLT_MQ_CASE(8)
        RLT_MQ_CASE(9)
        RLT_MQ_CASE(10)
        RLT_MQ_CASE(11)
        RLT_MQ_CASE(12)
        RLT_MQ_CASE(13)
        RLT_MQ_CASE(14)
        RLT_MQ_CASE(15)
        RLT_MQ_CASE(16)
#undef RLT_MQ_CASE
    }
    if (ok) rlt_count_launch();
    return ok;
}
template bool launch_attn_mq<true>(const bf16*, size_t, int, const int32_t*, int, bf16*, int, int,
                                   int, int, const ProjIn&, cudaStream_t);
template bool launch_attn_mq<false>(const bf16*, size_t, int, const int32_t*, int, bf16*, int,
                                    int, int, int, const ProjIn&, cudaStream_t);

}  // namespace rlt
