// C[M,N] = A[M,K] . W[N,K]^T on CUDA cores, fp32 accumulation.
//
// The plain fallback GEMM: fp32 models (no fp32 tensor-core path is used) and
// shapes the tensor-core kernel does not take.  Every output element sums its
// K products in ascending k, independently of M and N, so a row's result
// does not depend on the batch it is computed in.
#include "kernels.cuh"

namespace rlt {

namespace {
constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <typename T, int MODE>
__global__ void __launch_bounds__(NT)
k_gemm_simt(const T* __restrict__ A, int lda, const T* __restrict__ W, int ldw,
            float* __restrict__ C, int ldc, T* __restrict__ Ct, int ldct, int M, int N, int K) {
    pdl_enter();
    __shared__ float As[BK][BM + 4];
    __shared__ float Ws[BK][BN + 4];
    int tid = threadIdx.x;
    int tx = tid % 16, ty = tid / 16;
    int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
        for (int q = 0; q < (BM * BK) / NT; ++q) {
            int e = tid + q * NT;
            int rr = e / BK, kk = e % BK;
            int gm = m0 + rr, gk = k0 + kk;
            As[kk][rr] = (gm < M && gk < K) ? to_f(A[(size_t)gm * lda + gk]) : 0.f;
            int gn = n0 + rr;
            Ws[kk][rr] = (gn < N && gk < K) ? to_f(W[(size_t)gn * ldw + gk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int gm = m0 + ty * 4 + i;
        if (gm >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int gn = n0 + tx * 4 + j;
            if (gn >= N) continue;
            if (MODE == kStoreF32) C[(size_t)gm * ldc + gn] = acc[i][j];
            else if (MODE == kAddF32) C[(size_t)gm * ldc + gn] += acc[i][j];
            else Ct[(size_t)gm * ldct + gn] = from_f<T>(acc[i][j]);
        }
    }
}
}  // namespace

template <typename T>
void launch_gemm_simt(const T* A, int lda, const T* W, int ldw, float* C, int ldc, T* Ct,
                      int ldct, int M, int N, int K, int mode, cudaStream_t st) {
    if (M <= 0 || N <= 0) return;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
    if (mode == kStoreF32)
        launch(k_gemm_simt<T, kStoreF32>, grid, NT, 0, st, A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K);
    else if (mode == kAddF32)
        launch(k_gemm_simt<T, kAddF32>, grid, NT, 0, st, A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K);
    else
        launch(k_gemm_simt<T, kStoreT>, grid, NT, 0, st, A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K);
    rlt_count_launch();
}

template void launch_gemm_simt<float>(const float*, int, const float*, int, float*, int, float*,
                                      int, int, int, int, int, cudaStream_t);
template void launch_gemm_simt<bf16>(const bf16*, int, const bf16*, int, float*, int, bf16*,
                                     int, int, int, int, int, cudaStream_t);

}  // namespace rlt
