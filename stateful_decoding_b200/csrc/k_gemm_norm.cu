// A residual projection and the RMSNorm that follows it, in one kernel:
//   z[M, N] += A[M, K] . W[N, K]^T,   Y = RMSNorm(z) * gain   (N = d)
// (greeksharifa "Recurrent Looped Transformer 요약 설명" §2.5 and jiphyeonjeon
// review "Recurrent Looped Transformer" §3.3: pre-norm residual blocks, each
// sublayer's output added to z and the next sublayer reading RMSNorm(z)).
//
// A cluster of CL = N / BN CTAs (at most 8) covers the whole width of 128
// rows: CTA c computes columns [c·BN, c·BN + BN) over the full K range with
// the tcgen05 pipeline of k_gemm_tc (warp 0 TMA, warp 1 MMA, warps 2-5
// epilogue).  Each epilogue thread owns one row: it adds its accumulator to
// z, stores z, and sends its partial sum of squares to every CTA of the
// cluster through distributed shared memory; after one cluster barrier it
// sums the CL partials in rank order and writes its slice of Y.  Waits are
// bounded; every thread reaches both cluster barriers whatever happened, and
// a CTA frees its tensor memory before it exits.
#include <cuda.h>

#include "fused.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

constexpr int BM = 128, BK = 64, STAGES = 4, NTHREADS = 192, MAXCL = 8;

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_peer_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

template <int BN>
constexpr uint32_t stage_bytes() { return (uint32_t)(BM * BK * 2 + BN * BK * 2); }
template <int BN>
constexpr size_t smem_bytes() { return (size_t)STAGES * stage_bytes<BN>() + 1024; }

template <int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
k_gemm_norm(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
            float* __restrict__ Z, const float* __restrict__ gain, bf16* __restrict__ Y, int M,
            int N, int K, float eps, int* err) {
    using namespace tc;
    constexpr uint32_t A_BYTES = BM * BK * 2, STAGE = stage_bytes<BN>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[STAGES], empty[STAGES], accum;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ float red[MAXCL][BM];           // partial sums of squares, by sender rank

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int nk = K / BK;
    const int CL = N / BN;
    const uint32_t rank = cluster_ctarank();

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
    if (warp == 1) tmem_alloc(&tmem_base, BN);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tmem_base;
    // every CTA of the cluster is running before any writes into a peer
    cluster_sync_all();
    // weight tiles never depend on the previous kernel: request them first
    const int pre = min(nk, STAGES);
    if (warp == 0 && lane == 0) {
        for (int kt = 0; kt < pre; ++kt) {
            mbar_expect_tx(&full[kt], STAGE);
            tma_load_2d(smem + kt * STAGE + A_BYTES, &tb, kt * BK, n0, &full[kt]);
        }
    }
    pdl_enter();

    const int q = warp & 3;
    const int r = 32 * q + lane, row = m0 + r;
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
                    tma_load_2d(smem + s * STAGE + A_BYTES, &tb, kt * BK, n0, &full[s]);
                }
                tma_load_2d(smem + s * STAGE, &ta, kt * BK, m0, &full[s]);
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
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    mma_bf16(tmem, sdesc_k_sw128(a + kk * 32), sdesc_k_sw128(b + kk * 32), idesc,
                             (kt | kk) != 0);
                if (kt + STAGES < nk) mma_commit(&empty[s]);
            }
            if (ok) mma_commit(&accum);
        }
    } else {
        // ---- pass 1: z += acc (this CTA's columns), partial sum of squares
        const bool got = __all_sync(0xffffffffu, mbar_wait(&accum, 0));
        if (!got) abort_flag = 1;
        fence_after_sync();
        float ss = 0.f;
        if (got) {
            float* zr = Z + (size_t)row * N + n0;
#pragma unroll 1
            for (int c = 0; c < BN; c += 64) {
                float v[64];
                tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c, v);
                if (row < M) {
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        float4 z4 = *reinterpret_cast<const float4*>(zr + c + 4 * u);
                        z4.x += v[4 * u];
                        z4.y += v[4 * u + 1];
                        z4.z += v[4 * u + 2];
                        z4.w += v[4 * u + 3];
                        *reinterpret_cast<float4*>(zr + c + 4 * u) = z4;
                        ss += z4.x * z4.x + z4.y * z4.y + z4.z * z4.z + z4.w * z4.w;
                    }
                }
            }
        }
        // send the partial to every CTA of the cluster (slot = this CTA's rank)
        const uint32_t slot = smem_u32(&red[rank][r]);
        for (int p = 0; p < CL; ++p) st_peer_f32(map_peer(slot, (uint32_t)p), ss);
    }
    __syncwarp();               // the barrier below is warp-collective
    cluster_sync_all();         // every thread of every CTA, once

    if (warp >= 2 && !abort_flag && row < M) {
        // ---- pass 2: the row's sum of squares (rank order), Y slice
        float ss = 0.f;
        for (int p = 0; p < CL; ++p) ss += red[p][r];
        const float inv = 1.0f / sqrtf(ss / (float)N + eps);
        const float* zr = Z + (size_t)row * N + n0;
        bf16* yr = Y + (size_t)row * N + n0;
#pragma unroll 4
        for (int c = 0; c < BN; c += 8) {
            const float4 a = *reinterpret_cast<const float4*>(zr + c);
            const float4 b = *reinterpret_cast<const float4*>(zr + c + 4);
            const float4 ga = *reinterpret_cast<const float4*>(gain + n0 + c);
            const float4 gb = *reinterpret_cast<const float4*>(gain + n0 + c + 4);
            __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x * inv * ga.x, a.y * inv * ga.y);
            __nv_bfloat162 p1 = __floats2bfloat162_rn(a.z * inv * ga.z, a.w * inv * ga.w);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x * inv * gb.x, b.y * inv * gb.y);
            __nv_bfloat162 p3 = __floats2bfloat162_rn(b.z * inv * gb.z, b.w * inv * gb.w);
            uint4 w;
            w.x = *reinterpret_cast<uint32_t*>(&p0);
            w.y = *reinterpret_cast<uint32_t*>(&p1);
            w.z = *reinterpret_cast<uint32_t*>(&p2);
            w.w = *reinterpret_cast<uint32_t*>(&p3);
            *reinterpret_cast<uint4*>(yr + c) = w;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, BN);
    if (threadIdx.x == 0 && abort_flag) atomicExch(err, kDevTimeout);
}

template <int BN>
bool launch_bn(const bf16* A, int lda, const bf16* W, int ldw, float* Z, const float* gain,
               bf16* Y, int M, int N, int K, float eps, int* err, cudaStream_t st) {
    CUtensorMap ta, tb;
    if (!make_tma_2d_bf16(&ta, A, M, K, lda, BM) || !make_tma_2d_bf16(&tb, W, N, K, ldw, BN))
        return false;
    if (!set_smem_once(reinterpret_cast<const void*>(k_gemm_norm<BN>), smem_bytes<BN>()))
        return false;
    set_carveout_once(reinterpret_cast<const void*>(k_gemm_norm<BN>));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(N / BN, (M + BM - 1) / BM, 1);
    cfg.blockDim = dim3(NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<BN>();
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = N / BN;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, k_gemm_norm<BN>, ta, tb, Z, gain, Y, M, N, K, eps, err) !=
        cudaSuccess)
        return false;
    rlt_count_launch();
    return true;
}

}  // namespace

bool launch_gemm_norm(const bf16* A, int lda, const bf16* W, int ldw, float* Z, const float* gain,
                      bf16* Y, int M, int N, int K, float eps, int* err, cudaStream_t st) {
    if (M <= 0 || K < BK || K % BK || N % 64) return false;
    if (lda % 8 || ldw % 8 || ((uintptr_t)A & 15) || ((uintptr_t)W & 15)) return false;
    // the narrowest tile that keeps the cluster within 8 CTAs
    if (N <= 64 * MAXCL) return launch_bn<64>(A, lda, W, ldw, Z, gain, Y, M, N, K, eps, err, st);
    if (N <= 128 * MAXCL && N % 128 == 0)
        return launch_bn<128>(A, lda, W, ldw, Z, gain, Y, M, N, K, eps, err, st);
    if (N <= 256 * MAXCL && N % 256 == 0)
        return launch_bn<256>(A, lda, W, ldw, Z, gain, Y, M, N, K, eps, err, st);
    return false;
}

}  // namespace rlt
