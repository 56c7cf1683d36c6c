// GEMM dispatch: C[M,N] = A[M,K] . W[N,K]^T with the epilogues of GemmMode.
// bf16 goes to the tcgen05 kernel whenever its shape rules hold (K a multiple
// of 64, N >= 16, 16-byte aligned rows); fp32 and the remaining shapes use the
// CUDA-core kernel.  RLT_GEMM=simt forces the CUDA-core kernel (diagnostics).
#include <cstdlib>
#include <cstring>

#include "kernels.cuh"

namespace rlt {

bool launch_gemm_tc(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc, bf16* Ct,
                    int ldct, int M, int N, int K, int mode, cudaStream_t st);

static bool tc_enabled() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("RLT_GEMM");
        v = (e && strcmp(e, "simt") == 0) ? 0 : 1;
    }
    return v == 1;
}

template <>
void launch_gemm<float>(const float* A, int lda, const float* W, int ldw, float* C, int ldc,
                        float* Ct, int ldct, int M, int N, int K, int mode, cudaStream_t st) {
    launch_gemm_simt<float>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, st);
}

template <>
void launch_gemm<bf16>(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                       bf16* Ct, int ldct, int M, int N, int K, int mode, cudaStream_t st) {
    if (tc_enabled() && launch_gemm_tc(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, st))
        return;
    launch_gemm_simt<bf16>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, st);
}

}  // namespace rlt
