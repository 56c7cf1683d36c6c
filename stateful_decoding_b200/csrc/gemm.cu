// GEMM dispatch: C[M,N] = A[M,K] . W[N,K]^T with the epilogues of GemmMode.
#include "kernels.cuh"

namespace rlt {

template <typename T>
void launch_gemm(const T* A, int lda, const T* W, int ldw, float* C, int ldc, T* Ct, int ldct,
                 int M, int N, int K, int mode, cudaStream_t st) {
    launch_gemm_simt<T>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, st);
}

template void launch_gemm<float>(const float*, int, const float*, int, float*, int, float*, int,
                                 int, int, int, int, cudaStream_t);
template void launch_gemm<bf16>(const bf16*, int, const bf16*, int, float*, int, bf16*, int, int,
                                int, int, int, cudaStream_t);

}  // namespace rlt
