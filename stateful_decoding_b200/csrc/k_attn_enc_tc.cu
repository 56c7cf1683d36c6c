// The encoder's causal self-attention on the tensor cores (jiphyeonjeon
// review "Recurrent Looped Transformer" §3.2: the encoder runs in parallel
// over the known tokens; greeksharifa "Recurrent Looped Transformer 요약
// 설명" §2.2): for one (row, head) and a tile of 128 query positions,
// S = Q K^T over the head's cache prefix (at most 256 keys) into tensor
// memory, an exact two-pass softmax per query row, P in bf16 in shared
// memory, and O = P V on the tensor cores.
//
// d_h = 64.  One CTA of 4 warps per (row, head, 128 queries); warp w owns
// query rows 32w..32w+31 (its TMEM lane quarter).  Operands are staged by
// the threads in the K-major 128-byte-swizzled layout the MMA descriptors
// expect (row r of an 8-row atom keeps its 16-byte chunk c at c ^ (r % 8)):
// Q converted from fp32 to bf16, K copied, V transposed (rows = d_h, keys
// along K).  Keys past the CTA's last valid position are staged as zeros and
// masked by position.  q and the probabilities are bf16 at the MMA inputs
// (the decoder and the CUDA-core path keep them fp32); the row sum is taken
// over the rounded probabilities.  Waits are bounded; a timeout sets the
// state's error word and the CTA still frees its tensor memory.
#include <math.h>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

constexpr int EDH = 64;          // head size handled
constexpr int EQ = 128;          // query rows per CTA
constexpr int ENT = 128;         // threads

// byte offset of the 16-byte chunk `c` of row `r` in a swizzled K-major tile
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return (uint32_t)r * 128u + (uint32_t)((c ^ (r & 7)) << 4);
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ void proxy_fence() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int NK>
__global__ void __launch_bounds__(ENT)
k_attn_enc_tc(const float* __restrict__ Q, const bf16* __restrict__ cache, size_t row_stride,
              int T_cap, const int32_t* __restrict__ pos, bf16* __restrict__ A, int n, int heads,
              int* err) {
    using namespace tc;
    // shared memory: V^T [NK/64 blocks][64 rows][128 B] | K tiles + Q, later P
    constexpr uint32_t VT_BYTES = NK / 64 * 64 * 128;     // 8 KB per 64 keys
    constexpr uint32_t KT_BYTES = EQ * 128;               // one 128-key K tile, 16 KB
    constexpr uint32_t P_BLOCK = EQ * 128;                // 64 keys of P, 16 KB
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sVT = smem;
    uint8_t* sR2 = smem + VT_BYTES;            // K tiles at 0, Q after them; P over both
    uint8_t* sQ = sR2 + (NK / 128) * KT_BYTES;
    uint8_t* sP = sR2;
    __shared__ uint64_t bar_s, bar_o;
    __shared__ uint32_t tmem_base;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / heads, h = blockIdx.x % heads;
    const int q0 = blockIdx.y * EQ;
    const int nq = min(EQ, n - q0);
    const int d = heads * EDH;

    if (threadIdx.x == 0) {
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    pdl_enter();

    const int p0 = pos[b];
    const int kvalid = min(p0 + q0 + nq, NK);       // keys this CTA may attend to
    const bf16* kg = cache + (size_t)b * row_stride + (size_t)h * T_cap * EDH;
    const bf16* vg = kg + (size_t)heads * T_cap * EDH;

    // ---- stage Q (fp32 -> bf16), K, V^T: each thread issues all its loads
    // of a phase before its first store
    {
        constexpr int QI = EQ * 8 / ENT;           // 16-byte bf16 chunks of Q per thread
        float4 qa[QI], qb[QI];
#pragma unroll
        for (int u = 0; u < QI; ++u) {
            const int e = threadIdx.x + u * ENT, r = e >> 3, c = e & 7;
            qa[u] = qb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < nq) {
                const float* src = Q + (size_t)(b * n + q0 + r) * d + h * EDH + c * 8;
                qa[u] = *reinterpret_cast<const float4*>(src);
                qb[u] = *reinterpret_cast<const float4*>(src + 4);
            }
        }
#pragma unroll
        for (int u = 0; u < QI; ++u) {
            const int e = threadIdx.x + u * ENT, r = e >> 3, c = e & 7;
            *reinterpret_cast<uint4*>(sQ + sw128(r, c)) =
                make_uint4(pack2(qa[u].x, qa[u].y), pack2(qa[u].z, qa[u].w), pack2(qb[u].x, qb[u].y),
                           pack2(qb[u].z, qb[u].w));
        }
    }
    {
        constexpr int KI = NK * 8 / ENT;           // 16-byte chunks of K per thread
        uint4 kv[KI];
#pragma unroll
        for (int u = 0; u < KI; ++u) {
            const int e = threadIdx.x + u * ENT, k = e >> 3, c = e & 7;
            kv[u] = make_uint4(0, 0, 0, 0);
            if (k < kvalid) kv[u] = *reinterpret_cast<const uint4*>(kg + (size_t)k * EDH + c * 8);
        }
#pragma unroll
        for (int u = 0; u < KI; ++u) {
            const int e = threadIdx.x + u * ENT, k = e >> 3, c = e & 7;
            *reinterpret_cast<uint4*>(sR2 + (k >> 7) * KT_BYTES + sw128(k & 127, c)) = kv[u];
        }
    }
    // V^T: a thread takes 8 consecutive keys of one 8-wide column chunk and
    // writes them as 8 rows (one per d_h index) of 8 keys each
#pragma unroll
    for (int e = threadIdx.x; e < (NK / 8) * 8; e += ENT) {
        const int kgrp = e >> 3, c = e & 7;        // keys 8*kgrp .. +7, d_h 8c .. 8c+7
        uint32_t in[8][4];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int k = kgrp * 8 + kk;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (k < kvalid) w = *reinterpret_cast<const uint4*>(vg + (size_t)k * EDH + c * 8);
            in[kk][0] = w.x;
            in[kk][1] = w.y;
            in[kk][2] = w.z;
            in[kk][3] = w.w;
        }
        const int k0 = kgrp * 8, blk = k0 >> 6, kc = (k0 & 63) >> 3;
#pragma unroll
        for (int x8 = 0; x8 < 8; ++x8) {           // d_h index c*8 + x8
            const int sh = (x8 & 1) * 16, wd = x8 >> 1;
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t lo = (in[2 * j][wd] >> sh) & 0xFFFFu;
                const uint32_t hi = (in[2 * j + 1][wd] >> sh) & 0xFFFFu;
                o[j] = lo | (hi << 16);
            }
            const int row = c * 8 + x8;
            *reinterpret_cast<uint4*>(sVT + blk * (64 * 128) + sw128(row, kc)) =
                make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    proxy_fence();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ---- S = Q K^T: NK/128 MMA groups of N = 128 keys into TMEM columns
    bool ok = true;
    if (threadIdx.x == 0) {
        constexpr uint32_t idS = idesc_bf16(EQ, 128);
        const uint32_t aq = smem_u32(sQ);
#pragma unroll
        for (int kt = 0; kt < NK / 128; ++kt) {
            const uint32_t bk = smem_u32(sR2 + kt * KT_BYTES);
#pragma unroll
            for (int kk = 0; kk < EDH / 16; ++kk)
                mma_bf16(tmem + kt * 128, sdesc_k_sw128(aq + kk * 32), sdesc_k_sw128(bk + kk * 32),
                         idS, kk != 0);
        }
        mma_commit(&bar_s);
    }
    if (!mbar_wait(&bar_s, 0)) ok = false;
    // tcgen05.ld is warp-collective: every lane of a warp takes the same path
    ok = __all_sync(0xffffffffu, ok);
    fence_after_sync();

    // ---- softmax of row r (exact: max, then exp and sum), P -> smem bf16
    const int r = 32 * warp + lane;
    const int qpos = p0 + 1 + q0 + r;               // 1-based; keys 0 .. qpos-1 visible
    const int nvis = r < nq ? min(qpos, NK) : 0;
    const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
    const float sc = 1.0f / sqrtf((float)EDH);
    // 64 columns of S per TMEM load (one wait each)
    float m = -INFINITY;
    if (ok) {
#pragma unroll 1
        for (int c = 0; c < NK; c += 64) {
            float v[64];
            tmem_ld64(trow + (uint32_t)c, v);
#pragma unroll
            for (int j = 0; j < 64; ++j)
                if (c + j < nvis) m = fmaxf(m, v[j] * sc);
        }
    }
    float sum = 0.f;
    if (ok) {
#pragma unroll 1
        for (int c = 0; c < NK; c += 64) {
            float v[64];
            tmem_ld64(trow + (uint32_t)c, v);
            uint8_t* pb = sP + (c >> 6) * P_BLOCK;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {          // 8 keys per 16-byte chunk
                uint32_t w[4];
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    const int k = 8 * ch + j;
                    const float e0 = (c + k < nvis) ? __expf(v[k] * sc - m) : 0.f;
                    const float e1 = (c + k + 1 < nvis) ? __expf(v[k + 1] * sc - m) : 0.f;
                    __nv_bfloat162 p2 = __floats2bfloat162_rn(e0, e1);
                    sum += __low2float(p2) + __high2float(p2);
                    w[j / 2] = *reinterpret_cast<uint32_t*>(&p2);
                }
                *reinterpret_cast<uint4*>(pb + sw128(r, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    proxy_fence();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    // ---- O = P V: K = NK keys, N = 64, into TMEM columns 0..63 (S is consumed)
    if (threadIdx.x == 0) {
        if (ok) {
            constexpr uint32_t idO = idesc_bf16(EQ, EDH);
#pragma unroll
            for (int kc = 0; kc < NK / 16; ++kc) {
                const uint32_t ap = smem_u32(sP + (kc >> 2) * P_BLOCK) + (kc & 3) * 32;
                const uint32_t bv = smem_u32(sVT + (kc >> 2) * (64 * 128)) + (kc & 3) * 32;
                mma_bf16(tmem, sdesc_k_sw128(ap), sdesc_k_sw128(bv), idO, kc != 0);
            }
        }
        mma_commit(&bar_o);
    }
    if (!mbar_wait(&bar_o, 0)) ok = false;
    ok = __all_sync(0xffffffffu, ok);
    fence_after_sync();
    if (ok) {
        // all lanes load (warp-collective); rows past the block store nothing
        const float inv = r < nq ? 1.0f / sum : 0.f;
        bf16* dst = A + (size_t)(b * n + q0 + min(r, nq - 1)) * d + h * EDH;
        float v[64];
        tmem_ld64(trow, v);                       // the whole output row (d_h = 64)
        if (r < nq) {
#pragma unroll
            for (int c = 0; c < EDH; c += 8) {
                *reinterpret_cast<uint4*>(dst + c) =
                    make_uint4(pack2(v[c] * inv, v[c + 1] * inv), pack2(v[c + 2] * inv, v[c + 3] * inv),
                               pack2(v[c + 4] * inv, v[c + 5] * inv), pack2(v[c + 6] * inv, v[c + 7] * inv));
            }
        }
    }
    if (!ok && threadIdx.x == 0) atomicExch(err, kDevTimeout);
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

template <int NK>
bool launch_nk(const float* Q, const bf16* cache, size_t row_stride, int T_cap, const int32_t* pos,
               bf16* A, int B, int n, int heads, int* err, cudaStream_t st) {
    constexpr size_t smem = (size_t)NK / 64 * 64 * 128 + (NK / 128) * EQ * 128 + EQ * 128 + 1024;
    constexpr size_t smem_p = (size_t)NK / 64 * 64 * 128 + (size_t)NK / 64 * EQ * 128 + 1024;
    constexpr size_t bytes = smem > smem_p ? smem : smem_p;
    if (!set_smem_once(reinterpret_cast<const void*>(k_attn_enc_tc<NK>), bytes)) return false;
    launch(k_attn_enc_tc<NK>, dim3(B * heads, (n + EQ - 1) / EQ), ENT, bytes, st, Q, cache,
           row_stride, T_cap, pos, A, n, heads, err);
    rlt_count_launch();
    return true;
}

}  // namespace

bool launch_attn_enc_tc(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
                        const int32_t* pos, bf16* A, int B, int n, int heads, int dh, int max_keys,
                        int* err, cudaStream_t st) {
    if (B * n <= 0) return false;
    // longer prefixes and d_h = 128: key tiles with a running softmax
    if (dh != EDH || max_keys > 256)
        return launch_attn_enc_fa(Q, cache, row_stride, T_cap, pos, A, B, n, heads, dh, err, st);
    if (max_keys <= 128)
        return launch_nk<128>(Q, cache, row_stride, T_cap, pos, A, B, n, heads, err, st);
    return launch_nk<256>(Q, cache, row_stride, T_cap, pos, A, B, n, heads, err, st);
}

}  // namespace rlt
