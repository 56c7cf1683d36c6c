// C[M,N] = A[M,K] . W[N,K]^T on the 5th-generation tensor cores (tcgen05),
// bf16 operands, fp32 accumulation in tensor memory.
//
// One CTA computes a 128 x BN tile.  Warp 0 streams K-slices of A and W into
// a 4-stage shared-memory ring with TMA (128-byte swizzle); one thread of
// warp 1 issues the MMAs (4 per 64-wide K-slice) and releases each stage with
// tcgen05.commit; warps 2-5 wait for the final commit, read the accumulator
// out of TMEM (each warp its 32-lane quarter) and apply the epilogue.  Every
// wait is bounded: a wait that gives up records a timeout in the device error
// word, and the CTA still frees its TMEM and exits.
//
// Each output element sums its K products in the same order whatever M, N
// and the tile position, so a row's result does not depend on its batch.
#include <cuda.h>

#include <cstdlib>
#include <cstring>

#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {

__device__ int g_dev_error;   // sticky: set by kernels that give up a bounded wait

int read_and_clear_device_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        int z = 0;
        cudaMemcpyToSymbol(g_dev_error, &z, sizeof(int));
    }
    return v;
}

namespace {

constexpr int BM = 128, BK = 64, STAGES = 4, NTHREADS = 192;

template <int BN>
constexpr uint32_t stage_bytes() { return (uint32_t)(BM * BK * 2 + BN * BK * 2); }
// TMEM allocations are powers of two of at least 32 columns
__host__ __device__ constexpr uint32_t tmem_cols(int n) {
    return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : n <= 256 ? 256u : 512u;
}
template <int BN>
constexpr size_t smem_bytes() { return (size_t)STAGES * stage_bytes<BN>() + 1024; }

template <int BN, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
          float* __restrict__ C, int ldc, bf16* __restrict__ Ct, int ldct, int M, int N, int K,
          int cps, size_t slab, int tsplit) {
    using namespace tc;
    constexpr uint32_t A_BYTES = BM * BK * 2, STAGE = stage_bytes<BN>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[STAGES], empty[STAGES], accum;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    // split-K: this CTA sums K-chunks [kbeg, kbeg+nk) and, with several
    // splits, writes its partial sums to slab blockIdx.z of C.  With tsplit
    // > 1 the CTA takes every K-chunk instead, sums each run of cps chunks in
    // its own TMEM accumulator, and its epilogue adds the runs in run order
    // -- the sum a consumer of tsplit slabs forms -- into one slab.
    const int kbeg = tsplit > 1 ? 0 : blockIdx.z * cps;
    const int nk = tsplit > 1 ? K / BK : min(K / BK - kbeg, cps);
    C += (size_t)blockIdx.z * slab;
    const uint32_t tcols = tmem_cols(BN * tsplit);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&accum, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_map(&ta);
        prefetch_map(&tb);
    }
    if (warp == 1) tmem_alloc(&tmem_base, tcols);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    // The set-up above and the first stages' weight tiles (weights are never
    // written by a kernel) overlap the previous kernel of the stream; the
    // activations are read only after it has finished.
    const int pre = min(nk, STAGES);
    if (warp == 0 && lane == 0) {
        for (int kt = 0; kt < pre; ++kt) {
            mbar_expect_tx(&full[kt], STAGE);
            tma_load_2d(smem + kt * STAGE + A_BYTES, &tb, (kbeg + kt) * BK, n0, &full[kt]);
        }
    }
    pdl_enter();

    if (warp == 0) {
        if (lane == 0) {
            for (int kt = 0; kt < nk; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (kt >= STAGES && !mbar_wait(&empty[s], ph ^ 1u)) {
                    abort_flag = 1;
                    break;
                }
                if (kt >= pre) {
                    mbar_expect_tx(&full[s], STAGE);
                    tma_load_2d(smem + s * STAGE + A_BYTES, &tb, (kbeg + kt) * BK, n0, &full[s]);
                }
                tma_load_2d(smem + s * STAGE, &ta, (kbeg + kt) * BK, m0, &full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BM, BN);
            bool ok = true;
            for (int kt = 0; kt < nk; ++kt) {
                const int s = kt % STAGES;
                const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
                if (!mbar_wait(&full[s], ph)) {
                    abort_flag = 1;
                    ok = false;
                    break;
                }
                const uint32_t a = smem_u32(smem + s * STAGE), b = a + A_BYTES;
                // run of this chunk (tsplit > 1): its own accumulator, restarted
                // at the run's first chunk
                const int run = tsplit > 1 ? kt / cps : 0;
                const int kin = kt - run * cps;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    mma_bf16(tmem + (uint32_t)(run * BN), sdesc_k_sw128(a + kk * 32),
                             sdesc_k_sw128(b + kk * 32), idesc, (kin | kk) != 0);
                // release the stage only if the producer will refill it
                if (kt + STAGES < nk) mma_commit(&empty[s]);
            }
            if (ok) mma_commit(&accum);
        }
    } else {
        if (MODE == kSwiGLU) {
            // columns come in 64-wide groups (kW13Block = 32): 32 gates, then
            // the 32 matching up projections; unit u of group g0 goes to Ct
            // column (n0+g0)/2+u
            if (mbar_wait(&accum, 0)) {
                fence_after_sync();
                const int q = warp & 3;
                const int row = m0 + 32 * q + lane;
                const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
                for (int g0 = 0; g0 < BN; g0 += 2 * kW13Block) {
                    {
                        const int c = 0;
                        float a[32], u[32];
                        tmem_ld32(tq + (uint32_t)g0, a);
                        tmem_ld32(tq + (uint32_t)(g0 + kW13Block), u);
                        if (row < M && n0 + g0 + 2 * kW13Block <= N) {
                            uint4* dst = reinterpret_cast<uint4*>(
                                Ct + (size_t)row * ldct + (n0 + g0) / 2 + c);
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
                                dst[h] = w;
                            }
                        }
                    }
                }
            } else {
                abort_flag = 1;
            }
        } else {
            const bool got = mbar_wait(&accum, 0);
            if (!got) abort_flag = 1;
            fence_after_sync();
            const int q = warp & 3;
            const int row = m0 + 32 * q + lane;
            const bool vec = MODE == kStoreT
                                 ? ((ldct & 7) == 0 && ((uintptr_t)Ct & 15) == 0)
                                 : ((ldc & 3) == 0 && ((uintptr_t)C & 15) == 0);
            if (BN <= 128 && vec && n0 + BN <= N) {
                // Whole-width narrow tile (the decoder's few-hundred-row
                // projections): stage the accumulator in shared memory (the
                // pipeline stages are free once the last MMA has completed), then
                // write it out row-contiguously, consecutive threads on
                // consecutive 16-byte pieces of a row.
                constexpr int SP = BN + 4;          // row pitch in floats (conflict-free)
                float* stg = reinterpret_cast<float*>(smem);
                const int r = 32 * q + lane;
                if (__all_sync(0xffffffffu, got)) {
#pragma unroll 1
                    for (int c = 0; c < BN; c += 64) {
                        float v[64];
                        tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c, v);
                        // later runs added in run order (v = ((P0 + P1) + P2) ...)
                        for (int run = 1; run < tsplit; ++run) {
                            float w[64];
                            tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) +
                                          (uint32_t)(run * BN + c), w);
#pragma unroll
                            for (int i = 0; i < 64; ++i) v[i] += w[i];
                        }
                        float4* d4 = reinterpret_cast<float4*>(stg + (size_t)r * SP + c);
#pragma unroll
                        for (int u = 0; u < 16; ++u)
                            d4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    }
                }
                // the four epilogue warps meet here whatever their waits said
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (abort_flag) goto epilogue_done;
                constexpr int C4 = BN / 4;
                const int et = threadIdx.x - 64;
                // RA pieces per thread and pass; to accumulate, their 8 pieces
                // of C are read ahead of the stores (a store could alias a
                // later load, so loads and stores would not overlap otherwise)
                constexpr int RA = MODE == kAddF32 ? 8 : 4;
#pragma unroll 1
                for (int i0 = et; i0 < BM * C4; i0 += RA * 128) {
                    float4 o[RA];
                    if (MODE == kAddF32) {
#pragma unroll
                        for (int u = 0; u < RA; ++u) {
                            const int i = i0 + u * 128, grow = m0 + i / C4;
                            o[u] = (i < BM * C4 && grow < M)
                                       ? *reinterpret_cast<const float4*>(
                                             C + (size_t)grow * ldc + n0 + 4 * (i % C4))
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < RA; ++u) {
                        const int i = i0 + u * 128;
                        const int rr = i / C4, c4 = i % C4, grow = m0 + rr;
                        if (i >= BM * C4 || grow >= M) continue;
                        float4 w = *reinterpret_cast<const float4*>(stg + (size_t)rr * SP + 4 * c4);
                        if (MODE == kStoreT) {
                            __nv_bfloat162 a = __floats2bfloat162_rn(w.x, w.y);
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(w.z, w.w);
                            uint2 u2;
                            u2.x = *reinterpret_cast<uint32_t*>(&a);
                            u2.y = *reinterpret_cast<uint32_t*>(&b2);
                            *reinterpret_cast<uint2*>(Ct + (size_t)grow * ldct + n0 + 4 * c4) = u2;
                        } else {
                            float4* dst = reinterpret_cast<float4*>(C + (size_t)grow * ldc + n0 + 4 * c4);
                            if (MODE == kAddF32) {
                                w.x += o[u].x;
                                w.y += o[u].y;
                                w.z += o[u].z;
                                w.w += o[u].w;
                            }
                            *dst = w;
                        }
                    }
                }
            } else if (__all_sync(0xffffffffu, got))
#pragma unroll 1
            for (int c64 = 0; c64 < BN; c64 += 64) {
            float v64[64];
            tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c64, v64);
#pragma unroll
            for (int c = c64; c < c64 + 64; c += 16) {
                const float* v = v64 + (c - c64);
                if (row < M) {
                    const int col0 = n0 + c;
                    if (vec && col0 + 16 <= N) {
                        // 16 consecutive outputs of this row: 16-byte stores
                        if (MODE == kStoreT) {
                            uint4* dst = reinterpret_cast<uint4*>(Ct + (size_t)row * ldct + col0);
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                uint4 w;
                                uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
                                for (int k = 0; k < 4; ++k) {
                                    __nv_bfloat162 p2 =
                                        __floats2bfloat162_rn(v[8 * u + 2 * k], v[8 * u + 2 * k + 1]);
                                    wp[k] = *reinterpret_cast<uint32_t*>(&p2);
                                }
                                dst[u] = w;
                            }
                        } else {
                            float4* dst = reinterpret_cast<float4*>(C + (size_t)row * ldc + col0);
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                float4 w = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2],
                                                       v[4 * u + 3]);
                                if (MODE == kAddF32) {
                                    const float4 o = dst[u];
                                    w.x += o.x;
                                    w.y += o.y;
                                    w.z += o.z;
                                    w.w += o.w;
                                }
                                dst[u] = w;
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int col = col0 + j;
                            if (col < N) {
                                if (MODE == kStoreF32) C[(size_t)row * ldc + col] = v[j];
                                else if (MODE == kAddF32) C[(size_t)row * ldc + col] += v[j];
                                else Ct[(size_t)row * ldct + col] = __float2bfloat16_rn(v[j]);
                            }
                        }
                    }
                }
            }
            }
        }
    }
epilogue_done:
    fence_before_sync();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, tcols);
    if (threadIdx.x == 0 && abort_flag) atomicExch(&g_dev_error, kDevTimeout);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D bf16 map over a row-major [rows][cols] matrix with row pitch `ld`
// elements; box = 64 columns (128 bytes, swizzled) x box_rows rows.
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// in_tmem: the split runs stay in one CTA's tensor memory (see the kernel)
template <int BN, int MODE>
bool launch_tc(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc, bf16* Ct,
               int ldct, int M, int N, int K, int splits, size_t slab, cudaStream_t st,
               bool in_tmem = false) {
    CUtensorMap ta, tb;
    if (!make_map(&ta, A, M, K, lda, BM) || !make_map(&tb, W, N, K, ldw, BN)) return false;
    if (!set_smem_once(reinterpret_cast<const void*>(k_gemm_tc<BN, MODE>), smem_bytes<BN>()))
        return false;
    const int nk = K / BK, cps = (nk + splits - 1) / splits, runs = (nk + cps - 1) / cps;
    if (in_tmem && BN * runs > 512) return false;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, in_tmem ? 1 : runs);
    launch(k_gemm_tc<BN, MODE>, grid, NTHREADS, smem_bytes<BN>(), st, ta, tb, C, ldc, Ct, ldct, M, N,
           K, cps, slab, in_tmem ? runs : 1);
    rlt_count_launch();
    return true;
}

template <int BN>
bool launch_tc_mode(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc, bf16* Ct,
                    int ldct, int M, int N, int K, int mode, int splits, size_t slab,
                    cudaStream_t st) {
    if (mode == kStoreF32)
        return launch_tc<BN, kStoreF32>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, splits, slab, st);
    if (splits != 1) return false;          // partial sums only go to fp32 slabs
    if (mode == kSwiGLU) {
        if constexpr (BN % (2 * kW13Block) == 0)
            return launch_tc<BN, kSwiGLU>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, 1, 0, st);
        return false;
    }
    if (mode == kAddF32)
        return launch_tc<BN, kAddF32>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, 1, 0, st);
    return launch_tc<BN, kStoreT>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, 1, 0, st);
}

}  // namespace

bool make_tma_2d_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld,
                      int box_rows) {
    return make_map(map, base, rows, cols, ld, box_rows);
}

bool launch_gemm_persist(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                         bf16* Ct, int ldct, int M, int N, int K, int mode, cudaStream_t st);
bool persist_gemm_enabled() {
    static const bool on = [] {
        const char* e = getenv("RLT_GEMM_PERSIST");
        return !(e && strcmp(e, "0") == 0);
    }();
    return on;
}

// A split product of many rows in one slab: 64-wide tiles, every CTA over
// the whole K range with the split runs in separate TMEM accumulators, added
// in run order in the epilogue -- bit for bit the sum a consumer of the
// split's slabs forms, without the slabs.  False when it does not apply.
bool launch_gemm_tc_runs(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                         int M, int N, int K, int splits, cudaStream_t st) {
    if (M <= 0 || N < 16 || K < BK || K % BK || splits < 2) return false;
    if (lda % 8 || ldw % 8 || ((uintptr_t)A & 15) || ((uintptr_t)W & 15)) return false;
    if ((ldc & 3) || ((uintptr_t)C & 15) || N % 64) return false;
    return launch_tc<64, kStoreF32>(A, lda, W, ldw, C, ldc, nullptr, 0, M, N, K, splits, 0, st,
                                    true);
}

// Returns false (and launches nothing) when the shape or alignment does not
// suit the tensor-core kernel; the caller then uses the CUDA-core kernel.
bool launch_gemm_tc(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc, bf16* Ct,
                    int ldct, int M, int N, int K, int mode, int splits, size_t slab,
                    cudaStream_t st) {
    if (M <= 0 || N < 16 || K < BK || K % BK || splits < 1) return false;
    if (mode == kSwiGLU && (N % (2 * kW13Block) || (ldct % 8) || ((uintptr_t)Ct & 15)))
        return false;
    if (lda % 8 || ldw % 8 || ((uintptr_t)A & 15) || ((uintptr_t)W & 15)) return false;
    // many rows: the persistent kernel with two accumulators (epilogue of one
    // tile under the MMAs of the next); RLT_GEMM_PERSIST=0 turns it off
    if (M >= 2048 && splits == 1 && persist_gemm_enabled() &&
        launch_gemm_persist(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, st))
        return true;
    // wide tiles when M alone fills the machine, narrow ones (more CTAs)
    // otherwise; the SwiGLU epilogue needs whole 128-column gate/up groups
    if (M >= 2048)
        return launch_tc_mode<256>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, splits, slab, st);
    if (mode == kSwiGLU)        // 64-wide tiles: 32 gates and their 32 ups each
        return launch_tc_mode<64>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, 1, 0, st);
    return launch_tc_mode<64>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, splits, slab, st);
}

}  // namespace rlt
