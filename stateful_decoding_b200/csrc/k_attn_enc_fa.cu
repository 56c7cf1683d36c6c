// The encoder's causal self-attention over cache prefixes of any length, on
// the tensor cores (jiphyeonjeon review "Recurrent Looped Transformer" §3.2:
// the encoder runs in parallel over the known tokens; greeksharifa
// "Recurrent Looped Transformer 요약 설명" §2.2).  For one (row, head) and a
// tile of 128 query positions the keys 1..t are visited in tiles of 128:
// S = Q K^T into tensor memory, P in bf16 in shared memory, and O += P V
// accumulated in tensor memory across tiles.
//
// d_h = 64 or 128.  One CTA of 4 warps; thread r owns query row r (TMEM
// lane r).  Operands are staged by the threads in the K-major
// 128-byte-swizzled layout of the MMA descriptors: Q converted from fp32,
// K copied, V transposed (rows = d_h, keys along K).  Keys past the CTA's
// last query are staged as zeros and masked by position.
//
// Exact softmax in two passes over the key tiles: the first forms S tile by
// tile for each row's maximum m only; the second forms S again, the
// probabilities exp(s - m) rounded to bf16 (their sum l taken over the
// rounded values), and O += P V in tensor memory.  The rounding is therefore
// the short kernel's (k_attn_enc_tc.cu): q and the probabilities enter the
// MMAs as bf16, everything else stays fp32.  Waits are bounded; a timeout
// sets the state's error word, ends the key loops for the whole CTA, and the
// CTA still frees its tensor memory.
#include <math.h>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

constexpr int FQ = 128;              // query rows per CTA
constexpr int FK = 128;              // keys per tile
constexpr int FNT = 128;             // threads

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
template <int DH>
struct FaLayout {
    static constexpr int CH = DH / 64;                          // 64-wide chunks of d_h
    static constexpr uint32_t QK_CHUNK = 128 * 128;             // 128 rows x 128 B
    static constexpr uint32_t Q_BYTES = CH * QK_CHUNK;
    static constexpr uint32_t K_BYTES = CH * QK_CHUNK;
    static constexpr uint32_t VT_CHUNK = DH * 128;              // d_h rows x 64 keys
    static constexpr uint32_t VT_BYTES = (FK / 64) * VT_CHUNK;
    static constexpr uint32_t P_CHUNK = FQ * 128;               // 128 rows x 64 keys
    static constexpr uint32_t P_BYTES = (FK / 64) * P_CHUNK;
    static constexpr size_t SMEM = (size_t)Q_BYTES + K_BYTES + VT_BYTES + P_BYTES + 1024;
};

template <int DH>
__global__ void __launch_bounds__(FNT, 1)
k_attn_enc_fa(const float* __restrict__ Q, const bf16* __restrict__ cache, size_t row_stride,
              int T_cap, const int32_t* __restrict__ pos, bf16* __restrict__ A, int n, int heads,
              int* err) {
    using namespace tc;
    using L = FaLayout<DH>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + L::Q_BYTES;
    uint8_t* sVT = sK + L::K_BYTES;
    uint8_t* sP = sVT + L::VT_BYTES;
    __shared__ uint64_t bar_s, bar_o;
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / heads, h = blockIdx.x % heads;
    const int q0 = blockIdx.y * FQ;
    const int nq = min(FQ, n - q0);
    const int d = heads * DH;

    if (threadIdx.x == 0) {
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 0) tmem_alloc(&tmem_base, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;        // S: columns 0..127, O: 128..128+DH-1
    pdl_enter();

    const int p0 = pos[b];
    const int kvalid = p0 + q0 + nq;        // keys visible to the CTA's last query
    const int ntile = (kvalid + FK - 1) / FK;
    const bf16* kg = cache + (size_t)b * row_stride + (size_t)h * T_cap * DH;
    const bf16* vg = kg + (size_t)heads * T_cap * DH;

    // ---- Q (fp32 -> bf16), eight 16-byte chunks per thread per pass
    constexpr int QC = DH / 8;                       // chunks of 8 per row
#pragma unroll 1
    for (int e0 = 0; e0 < FQ * QC; e0 += FNT * 8) {
        float4 qa[8], qb[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + threadIdx.x + u * FNT, r = e / QC, c = e % QC;
            qa[u] = qb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < nq) {
                const float* src = Q + (size_t)(b * n + q0 + r) * d + h * DH + c * 8;
                qa[u] = *reinterpret_cast<const float4*>(src);
                qb[u] = *reinterpret_cast<const float4*>(src + 4);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + threadIdx.x + u * FNT, r = e / QC, c = e % QC;
            *reinterpret_cast<uint4*>(sQ + (c >> 3) * L::QK_CHUNK + sw128(r, c & 7)) =
                make_uint4(pack2(qa[u].x, qa[u].y), pack2(qa[u].z, qa[u].w),
                           pack2(qb[u].x, qb[u].y), pack2(qb[u].z, qb[u].w));
        }
    }

    const int r = 32 * warp + lane;
    const int qpos = p0 + 1 + q0 + r;               // keys 0 .. qpos-1 are visible
    const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
    const float sc = 1.0f / sqrtf((float)DH);
    bool ok = true;
    uint32_t s_uses = 0;                            // completed phases of bar_s

    // K tile of keys kb..kb+127: eight 16-byte chunks per thread per pass
    auto stage_k = [&](int kb) {
#pragma unroll 1
        for (int e0 = 0; e0 < FK * QC; e0 += FNT * 8) {
            uint4 kv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + threadIdx.x + u * FNT, k = e / QC, c = e % QC;
                kv[u] = make_uint4(0, 0, 0, 0);
                if (kb + k < kvalid)
                    kv[u] = *reinterpret_cast<const uint4*>(kg + (size_t)(kb + k) * DH + c * 8);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + threadIdx.x + u * FNT, k = e / QC, c = e % QC;
                *reinterpret_cast<uint4*>(sK + (c >> 3) * L::QK_CHUNK + sw128(k, c & 7)) = kv[u];
            }
        }
    };
    // V^T tile: a thread takes 8 consecutive keys of one 8-wide column chunk
    // and writes them as 8 rows (one per d_h index)
    auto stage_vt = [&](int kb) {
#pragma unroll 1
        for (int e = threadIdx.x; e < (FK / 8) * QC; e += FNT) {
            const int kgrp = e / QC, c = e % QC;
            uint32_t in[8][4];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int k = kb + kgrp * 8 + kk;
                uint4 w = make_uint4(0, 0, 0, 0);
                if (k < kvalid) w = *reinterpret_cast<const uint4*>(vg + (size_t)k * DH + c * 8);
                in[kk][0] = w.x;
                in[kk][1] = w.y;
                in[kk][2] = w.z;
                in[kk][3] = w.w;
            }
            const int k0 = kgrp * 8, blk = k0 >> 6, kc = (k0 & 63) >> 3;
#pragma unroll
            for (int x8 = 0; x8 < 8; ++x8) {
                const int sh = (x8 & 1) * 16, wd = x8 >> 1;
                uint32_t o[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint32_t lo = (in[2 * jj][wd] >> sh) & 0xFFFFu;
                    const uint32_t hi = (in[2 * jj + 1][wd] >> sh) & 0xFFFFu;
                    o[jj] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4*>(sVT + blk * L::VT_CHUNK + sw128(c * 8 + x8, kc)) =
                    make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    };
    // staged operands -> S = Q K^T (N = 128 keys) in TMEM columns 0..127;
    // false when the CTA gave up
    auto scores = [&]() -> bool {
        proxy_fence();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) return false;
        if (threadIdx.x == 0) {
            constexpr uint32_t idS = idesc_bf16(FQ, FK);
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
                const uint32_t a = smem_u32(sQ + (kk >> 2) * L::QK_CHUNK) + (kk & 3) * 32;
                const uint32_t bk = smem_u32(sK + (kk >> 2) * L::QK_CHUNK) + (kk & 3) * 32;
                mma_bf16(tmem, sdesc_k_sw128(a), sdesc_k_sw128(bk), idS, kk != 0);
            }
            mma_commit(&bar_s);
        }
        if (!mbar_wait(&bar_s, s_uses & 1u)) ok = false;
        ++s_uses;
        ok = __all_sync(0xffffffffu, ok);
        fence_after_sync();
        return true;
    };

    // ---- pass 1: each row's maximum scaled score over its visible keys
    float m = -INFINITY;
#pragma unroll 1
    for (int j = 0; j < ntile; ++j) {
        const int kb = j * FK;
        stage_k(kb);
        if (!scores()) break;
        const int nvis = r < nq ? min(max(qpos - kb, 0), FK) : 0;
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < FK; c += 64) {
                float v[64];
                tmem_ld64(trow + (uint32_t)c, v);
#pragma unroll
                for (int jj = 0; jj < 64; ++jj)
                    if (c + jj < nvis) m = fmaxf(m, v[jj] * sc);
            }
        }
        if (!ok) s_abort = 1;
        fence_before_sync();       // the TMEM reads finish before S is overwritten
    }

    // ---- pass 2: P = bf16(exp(s - m)), l = sum of P, O += P V
    float l = 0.f;
#pragma unroll 1
    for (int j = 0; j < ntile && !s_abort; ++j) {
        const int kb = j * FK;
        stage_k(kb);
        stage_vt(kb);
        if (!scores()) break;
        const int nvis = r < nq ? min(max(qpos - kb, 0), FK) : 0;
        float sum = 0.f;
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < FK; c += 64) {
                float v[64];
                tmem_ld64(trow + (uint32_t)c, v);
                uint8_t* pb = sP + (c >> 6) * L::P_CHUNK;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t w[4];
#pragma unroll
                    for (int jj = 0; jj < 8; jj += 2) {
                        const int k = 8 * ch + jj;
                        const float e0 = (c + k < nvis) ? __expf(v[k] * sc - m) : 0.f;
                        const float e1 = (c + k + 1 < nvis) ? __expf(v[k + 1] * sc - m) : 0.f;
                        __nv_bfloat162 p2 = __floats2bfloat162_rn(e0, e1);
                        sum += __low2float(p2) + __high2float(p2);
                        w[jj / 2] = *reinterpret_cast<uint32_t*>(&p2);
                    }
                    *reinterpret_cast<uint4*>(pb + sw128(r, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        l += sum;
        if (!ok) s_abort = 1;
        proxy_fence();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;

        // ---- O += P V (K = 128 keys, N = d_h) into TMEM columns 128..
        if (threadIdx.x == 0) {
            constexpr uint32_t idO = idesc_bf16(FQ, DH);
#pragma unroll
            for (int kc = 0; kc < FK / 16; ++kc) {
                const uint32_t ap = smem_u32(sP + (kc >> 2) * L::P_CHUNK) + (kc & 3) * 32;
                const uint32_t bv = smem_u32(sVT + (kc >> 2) * L::VT_CHUNK) + (kc & 3) * 32;
                mma_bf16(tmem + 128u, sdesc_k_sw128(ap), sdesc_k_sw128(bv), idO,
                         (j > 0 || kc > 0) ? 1u : 0u);
            }
            mma_commit(&bar_o);
        }
        if (!mbar_wait(&bar_o, (uint32_t)j & 1u)) ok = false;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) s_abort = 1;
        fence_after_sync();
    }
    __syncthreads();
    ok = ok && !s_abort;
    if (ok) {
        // all lanes load (warp-collective); rows past the block store nothing
        const float inv = r < nq ? 1.0f / l : 0.f;
        bf16* dst = A + (size_t)(b * n + q0 + min(r, nq - 1)) * d + h * DH;
#pragma unroll 1
        for (int c = 0; c < DH; c += 64) {
            float v[64];
            tmem_ld64(trow + 128u + (uint32_t)c, v);
            if (r < nq) {
#pragma unroll
                for (int x = 0; x < 64; x += 8)
                    *reinterpret_cast<uint4*>(dst + c + x) = make_uint4(
                        pack2(v[x] * inv, v[x + 1] * inv), pack2(v[x + 2] * inv, v[x + 3] * inv),
                        pack2(v[x + 4] * inv, v[x + 5] * inv), pack2(v[x + 6] * inv, v[x + 7] * inv));
            }
        }
    }
    if (!ok && threadIdx.x == 0) atomicExch(err, kDevTimeout);
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

template <int DH>
bool launch_fa(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
               const int32_t* pos, bf16* A, int B, int n, int heads, int* err, cudaStream_t st) {
    constexpr size_t bytes = FaLayout<DH>::SMEM;
    if (!set_smem_once(reinterpret_cast<const void*>(k_attn_enc_fa<DH>), bytes)) return false;
    launch(k_attn_enc_fa<DH>, dim3(B * heads, (n + FQ - 1) / FQ), FNT, bytes, st, Q, cache,
           row_stride, T_cap, pos, A, n, heads, err);
    rlt_count_launch();
    return true;
}

}  // namespace

bool launch_attn_enc_fa(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
                        const int32_t* pos, bf16* A, int B, int n, int heads, int dh, int* err,
                        cudaStream_t st) {
    if (B * n <= 0) return true;
    if (dh == 64) return launch_fa<64>(Q, cache, row_stride, T_cap, pos, A, B, n, heads, err, st);
    if (dh == 128)
        return launch_fa<128>(Q, cache, row_stride, T_cap, pos, A, B, n, heads, err, st);
    return false;
}

}  // namespace rlt
