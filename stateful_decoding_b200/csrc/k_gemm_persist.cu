// Large-M GEMM on the tensor cores (the encoder's projections over B·T rows):
// C[M,N] = A[M,K] . W[N,K]^T with a persistent grid and two accumulators.
//
// One CTA per SM loops over 128 x 256 output tiles (tile t: rows
// 128·(t / tiles_n), columns 256·(t % tiles_n)).  Warp 0 streams K-slices of
// A and W through a 4-stage TMA ring that runs on across tiles; one thread of
// warp 1 issues the MMAs of tile j into TMEM accumulator j % 2 (512 columns
// in all) and commits it; warps 2-5 drain accumulator j % 2 and apply the
// epilogue while the MMAs of tile j+1 already run into the other one.  The
// epilogues are those of k_gemm_tc (fp32 store, fp32 accumulate, SwiGLU over
// interleaved W1/W3 columns); each epilogue warp stages 32 rows x 32 columns
// at a time in shared memory and writes them row segment by row segment
// (128-byte coalesced stores; the accumulate mode reads z the same way).
// Each output element sums its K products in the
// same order as k_gemm_tc, whatever the tile's position.  Waits are bounded:
// a wait that gives up records a timeout in the device error word, the roles
// stop, and the CTA still frees its tensor memory.
#include <cuda.h>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, NTHREADS = 192;
constexpr uint32_t A_BYTES = BM * BK * 2, STAGE = BM * BK * 2 + BN * BK * 2;
// epilogue staging: each epilogue warp passes 32 rows x 32 columns of fp32
// through shared memory so that global stores cover whole row segments
constexpr int SPITCH = 36;                       // floats per staged row
constexpr uint32_t STG_WARP = 32 * SPITCH * 4;   // bytes per epilogue warp
constexpr size_t SMEM = (size_t)STAGES * STAGE + 4 * STG_WARP + 1024;

__device__ int g_persist_error;

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
k_gemm_persist(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
               float* __restrict__ C, int ldc, bf16* __restrict__ Ct, int ldct, int M, int N,
               int K, const RopeScatter rs) {
    using namespace tc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2];
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_n = N / BN, tiles = ((M + BM - 1) / BM) * tiles_n;
    const int nk = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);          // one arrival per epilogue warp
        }
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_map(&ta);
        prefetch_map(&tb);
    }
    if (warp == 1) tmem_alloc(&tmem_base, 2 * BN);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    pdl_enter();

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < tiles && !abort_flag; t += gridDim.x) {
                const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
                for (int kt = 0; kt < nk; ++kt, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (it >= STAGES && !mbar_wait(&empty[s], ph ^ 1u)) {
                        abort_flag = 1;
                        break;
                    }
                    mbar_expect_tx(&full[s], STAGE);
                    tma_load_2d(smem + s * STAGE, &ta, kt * BK, m0, &full[s]);
                    tma_load_2d(smem + s * STAGE + A_BYTES, &tb, kt * BK, n0, &full[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BM, BN);
            uint32_t it = 0;
            int j = 0;
            for (int t = blockIdx.x; t < tiles && !abort_flag; t += gridDim.x, ++j) {
                const int acc = j & 1;
                // the epilogue has drained this accumulator (tile j-2)
                if (j >= 2 && !mbar_wait(&tempty[acc], ((uint32_t)(j >> 1) & 1u) ^ 1u)) {
                    abort_flag = 1;
                    break;
                }
                fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kt = 0; kt < nk; ++kt, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(&full[s], ph)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a = smem_u32(smem + s * STAGE), b = a + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16(d, sdesc_k_sw128(a + kk * 32), sdesc_k_sw128(b + kk * 32), idesc,
                                 (kt | kk) != 0);
                    mma_commit(&empty[s]);
                }
                if (!ok) {
                    abort_flag = 1;
                    break;
                }
                mma_commit(&tfull[acc]);
            }
        }
    } else {
        const int q = warp & 3;
        int j = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            const int acc = j & 1;
            const bool got = __all_sync(0xffffffffu, !abort_flag &&
                                                          mbar_wait(&tfull[acc], (j >> 1) & 1u));
            if (!got) {
                abort_flag = 1;
                break;
            }
            fence_after_sync();
            const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
            const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * BN);
            // this warp's staging area: 32 rows x SPITCH floats
            float* stg = reinterpret_cast<float*>(smem + STAGES * STAGE + q * STG_WARP);
            const int rbase = m0 + 32 * q;             // first row of this warp
            if (MODE == kSwiGLU) {
                // 64-wide groups (kW13Block = 32): 32 gates, then their 32 ups
#pragma unroll 1
                for (int g0 = 0; g0 < BN; g0 += 2 * kW13Block) {
                    {
                        const int c = 0;
                        float a[32], u[32];
                        tmem_ld32(tq + (uint32_t)g0, a);
                        tmem_ld32(tq + (uint32_t)(g0 + kW13Block), u);
                        // 32 bf16 outputs of this row = 16 words, staged
                        uint32_t* srow = reinterpret_cast<uint32_t*>(stg) + lane * SPITCH;
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            uint4 w;
                            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int e = 8 * h + 2 * k;
                                const float y0 = silu_mul(a[e], u[e]);
                                const float y1 = silu_mul(a[e + 1], u[e + 1]);
                                __nv_bfloat162 p2 = __floats2bfloat162_rn(y0, y1);
                                wp[k] = *reinterpret_cast<uint32_t*>(&p2);
                            }
                            *reinterpret_cast<uint4*>(srow + 4 * h) = w;
                        }
                        __syncwarp();
                        // 4 lanes per row (16 bytes each): 8 rows per store
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int rr = 8 * k + (lane >> 2), c4 = lane & 3;
                            if (rbase + rr < M)
                                *reinterpret_cast<uint4*>(Ct + (size_t)(rbase + rr) * ldct +
                                                          (n0 + g0) / 2 + c + 8 * c4) =
                                    *reinterpret_cast<const uint4*>(
                                        reinterpret_cast<uint32_t*>(stg) + rr * SPITCH + 4 * c4);
                        }
                        __syncwarp();
                    }
                }
            } else if (MODE == kRopeScatter) {
                // the tile's 256 columns lie in one section: q, k or v
                const int sec = rs.sec0 + n0 / rs.d, c0 = n0 % rs.d;
                const int half = rs.dh >> 1, heads = rs.d / rs.dh;
                // the row of this lane's accumulator lane: its sequence and position
                const int row = rbase + lane;
                int rb = 0, rp = 1;
                if (row < M) {
                    rb = row / rs.n;
                    rp = __ldcg(rs.pos + rb) + 1 + row % rs.n;
                }
                uint32_t* stw = reinterpret_cast<uint32_t*>(stg);
                // q: 32 rotated values of this lane's row, staged, then written
                // as 128-byte row segments of Q (8 lanes per row)
                auto put_q = [&](const float (&x)[32], int col) {
                    float* srow = stg + lane * SPITCH;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<float4*>(srow + 4 * u) =
                            make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int rr = 4 * k + (lane >> 3), c4 = lane & 7;
                        if (rbase + rr < M)
                            *reinterpret_cast<float4*>(rs.Q + (size_t)(rbase + rr) * rs.d + col +
                                                       4 * c4) =
                                *reinterpret_cast<const float4*>(stg + rr * SPITCH + 4 * c4);
                    }
                    __syncwarp();
                };
#pragma unroll 1
                for (int hc = 0; hc < BN; hc += rs.dh) {
                    const int h = (c0 + hc) / rs.dh;
#pragma unroll 1
                    for (int j0 = 0; j0 < half; j0 += 32) {
                        // the pairs (j, j + d_h/2) for j = j0 .. j0+31 of head h
                        float x1[32], x2[32];
                        tmem_ld32(tq + (uint32_t)(hc + j0), x1);
                        tmem_ld32(tq + (uint32_t)(hc + half + j0), x2);
                        if (sec < 2 && row < M) {
                            const float* cs = rs.rope.cs + (size_t)rp * half + j0;
                            const float* sn = rs.rope.sn + (size_t)rp * half + j0;
#pragma unroll
                            for (int u = 0; u < 32; u += 4) {
                                const float4 c4 = __ldg(reinterpret_cast<const float4*>(cs + u));
                                const float4 s4 = __ldg(reinterpret_cast<const float4*>(sn + u));
                                rope_pair(x1[u], x2[u], c4.x, s4.x, x1[u], x2[u]);
                                rope_pair(x1[u + 1], x2[u + 1], c4.y, s4.y, x1[u + 1], x2[u + 1]);
                                rope_pair(x1[u + 2], x2[u + 2], c4.z, s4.z, x1[u + 2], x2[u + 2]);
                                rope_pair(x1[u + 3], x2[u + 3], c4.w, s4.w, x1[u + 3], x2[u + 3]);
                            }
                        }
                        if (sec == 0) {
                            put_q(x1, h * rs.dh + j0);
                            put_q(x2, h * rs.dh + half + j0);
                            continue;
                        }
                        // k or v, rounded to bf16: the row's two 64-byte pieces
                        // staged side by side, then 4 lanes per piece and row
                        {
                            uint32_t* srow = stw + lane * SPITCH;
#pragma unroll
                            for (int u = 0; u < 16; ++u) {
                                __nv_bfloat162 a2 = __floats2bfloat162_rn(x1[2 * u], x1[2 * u + 1]);
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(x2[2 * u], x2[2 * u + 1]);
                                srow[u] = *reinterpret_cast<uint32_t*>(&a2);
                                srow[16 + u] = *reinterpret_cast<uint32_t*>(&b2);
                            }
                        }
                        __syncwarp();
                        const size_t vofs = sec == 2 ? (size_t)heads * rs.T_cap * rs.dh : 0;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int rr = 8 * k + (lane >> 2), c4 = lane & 3;
                            const int br = __shfl_sync(0xffffffffu, rb, rr);
                            const int pr = __shfl_sync(0xffffffffu, rp, rr);
                            if (rbase + rr >= M) continue;
                            bf16* dst = rs.cache + (size_t)br * rs.row_stride + vofs +
                                        ((size_t)h * rs.T_cap + (pr - 1)) * rs.dh + j0 + 8 * c4;
                            *reinterpret_cast<uint4*>(dst) =
                                *reinterpret_cast<const uint4*>(stw + rr * SPITCH + 4 * c4);
                            *reinterpret_cast<uint4*>(dst + half) =
                                *reinterpret_cast<const uint4*>(stw + rr * SPITCH + 16 + 4 * c4);
                        }
                        __syncwarp();
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < BN; c += 64) {
                    // accumulate: this chunk's z values, all 16 loads in flight
                    // before the accumulator is read (8 lanes per row segment)
                    float4 o[2][8];
                    if (MODE == kAddF32) {
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                const int rr = 4 * k + (lane >> 3), c4 = lane & 7;
                                o[hf][k] = rbase + rr < M
                                               ? *reinterpret_cast<const float4*>(
                                                     C + (size_t)(rbase + rr) * ldc + n0 + c +
                                                     32 * hf + 4 * c4)
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                            }
                    }
                    float v[64];
                    tmem_ld64(tq + (uint32_t)c, v);
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float* srow = stg + lane * SPITCH;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<float4*>(srow + 4 * u) =
                                make_float4(v[32 * hf + 4 * u], v[32 * hf + 4 * u + 1],
                                            v[32 * hf + 4 * u + 2], v[32 * hf + 4 * u + 3]);
                        __syncwarp();
                        // 8 lanes per row (16 bytes each): 4 rows per store
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int rr = 4 * k + (lane >> 3), c4 = lane & 7;
                            if (rbase + rr >= M) continue;
                            float4 w = *reinterpret_cast<const float4*>(stg + rr * SPITCH + 4 * c4);
                            float4* dst = reinterpret_cast<float4*>(
                                C + (size_t)(rbase + rr) * ldc + n0 + c + 32 * hf + 4 * c4);
                            if (MODE == kAddF32) {
                                w.x += o[hf][k].x;
                                w.y += o[hf][k].y;
                                w.z += o[hf][k].z;
                                w.w += o[hf][k].w;
                            }
                            *dst = w;
                        }
                        __syncwarp();
                    }
                }
            }
            // this accumulator may take the MMAs of tile j+2
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 2 * BN);
    if (threadIdx.x == 0 && abort_flag) atomicExch(&g_persist_error, kDevTimeout);
}

template <int MODE>
bool launch_mode(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc, bf16* Ct,
                 int ldct, int M, int N, int K, cudaStream_t st, const RopeScatter& rs = {}) {
    CUtensorMap ta, tb;
    if (!make_tma_2d_bf16(&ta, A, M, K, lda, BM) || !make_tma_2d_bf16(&tb, W, N, K, ldw, BN))
        return false;
    if (!set_smem_once(reinterpret_cast<const void*>(k_gemm_persist<MODE>), SMEM)) return false;
    const int sms = sm_count();
    if (sms <= 0) return false;
    const int tiles = ((M + BM - 1) / BM) * (N / BN);
    launch(k_gemm_persist<MODE>, std::min(tiles, sms), NTHREADS, SMEM, st, ta, tb, C, ldc, Ct,
           ldct, M, N, K, rs);
    rlt_count_launch();
    return true;
}

}  // namespace

int read_and_clear_persist_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_persist_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        int z = 0;
        cudaMemcpyToSymbol(g_persist_error, &z, sizeof(int));
    }
    return v;
}

// Returns false (nothing launched) for shapes or modes it does not handle.
bool launch_gemm_persist(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                         bf16* Ct, int ldct, int M, int N, int K, int mode, cudaStream_t st) {
    if (M < 2048 || N % BN || K < BK || K % BK) return false;
    if (lda % 8 || ldw % 8 || ((uintptr_t)A & 15) || ((uintptr_t)W & 15)) return false;
    if (mode == kSwiGLU) {
        if (ldct % 8 || ((uintptr_t)Ct & 15)) return false;
        return launch_mode<kSwiGLU>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, st);
    }
    if (ldc % 4 || ((uintptr_t)C & 15)) return false;
    if (mode == kStoreF32)
        return launch_mode<kStoreF32>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, st);
    if (mode == kAddF32)
        return launch_mode<kAddF32>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, st);
    return false;
}

bool tc_gemm_enabled();
bool persist_gemm_enabled();

bool launch_gemm_rope_scatter(const bf16* A, int lda, const bf16* W, int ldw, int M, int N,
                              int K, const RopeScatter& rs, cudaStream_t st) {
    if (!tc_gemm_enabled() || !persist_gemm_enabled()) return false;
    if (M < 2048 || N % BN || K < BK || K % BK) return false;
    if (rs.d <= 0 || rs.d % BN || rs.n <= 0 || (rs.dh != 64 && rs.dh != 128)) return false;
    if (rs.sec0 < 0 || rs.sec0 > 1 || N != (3 - rs.sec0) * rs.d) return false;
    if (lda % 8 || ldw % 8 || ((uintptr_t)A & 15) || ((uintptr_t)W & 15)) return false;
    if (((uintptr_t)rs.cache & 15) || rs.row_stride % 8 || !rs.pos ||
        ((uintptr_t)rs.rope.cs & 15) || ((uintptr_t)rs.rope.sn & 15) || rs.rope.half != rs.dh / 2)
        return false;
    if (rs.sec0 == 0 && ((uintptr_t)rs.Q & 15)) return false;
    return launch_mode<kRopeScatter>(A, lda, W, ldw, nullptr, 0, nullptr, 0, M, N, K, st, rs);
}

}  // namespace rlt
