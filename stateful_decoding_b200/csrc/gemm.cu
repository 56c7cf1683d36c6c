// GEMM dispatch: C[M,N] = A[M,K] . W[N,K]^T with the epilogues of GemmMode.
// bf16 goes to the tcgen05 kernel whenever its shape rules hold (K a multiple
// of 64, N >= 16, 16-byte aligned rows); fp32 and the remaining shapes use the
// CUDA-core kernel.  RLT_GEMM=simt forces the CUDA-core kernel (diagnostics).
#include <cstdlib>
#include <cstring>

#include "kernels.cuh"

namespace rlt {

bool launch_gemm_tc(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc, bf16* Ct,
                    int ldct, int M, int N, int K, int mode, int splits, size_t slab,
                    cudaStream_t st);
bool launch_gemm_tc_runs(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                         int M, int N, int K, int splits, cudaStream_t st);

bool tc_gemm_enabled() {
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
    if (tc_gemm_enabled() && launch_gemm_tc(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, 1, 0, st))
        return;
    launch_gemm_simt<bf16>(A, lda, W, ldw, C, ldc, Ct, ldct, M, N, K, mode, st);
}

// Split-K partial sums: with `splits` > 1, slab z = C + z*slab holds the sum
// over the z-th run of K-chunks; the consumer adds the slabs in order.  The
// split count must depend on N and K only, never on M, so that a row's result
// does not depend on its batch.  From kRunsRows rows on, one slab holds the
// runs' sum already (the same additions in the same order, made in the GEMM's
// epilogue).  Returns the number of slabs written.
static constexpr int kRunsRows = 1024;
template <>
int launch_gemm_split<float>(const float* A, int lda, const float* W, int ldw, float* C, int ldc,
                             int M, int N, int K, int splits, size_t slab, cudaStream_t st) {
    (void)splits;
    (void)slab;
    launch_gemm_simt<float>(A, lda, W, ldw, C, ldc, nullptr, 0, M, N, K, kStoreF32, st);
    return 1;
}

template <>
int launch_gemm_split<bf16>(const bf16* A, int lda, const bf16* W, int ldw, float* C, int ldc,
                            int M, int N, int K, int splits, size_t slab, cudaStream_t st) {
    if (tc_gemm_enabled() && splits > 1 && K % 64 == 0) {
        const int nk = K / 64, cps = (nk + splits - 1) / splits, s = (nk + cps - 1) / cps;
        // enough rows to fill the machine without splitting CTAs: the runs
        // stay in tensor memory and one slab holds their ordered sum
        if (M >= kRunsRows && launch_gemm_tc_runs(A, lda, W, ldw, C, ldc, M, N, K, s, st))
            return 1;
        if (launch_gemm_tc(A, lda, W, ldw, C, ldc, nullptr, 0, M, N, K, kStoreF32, s, slab, st))
            return s;
    }
    launch_gemm<bf16>(A, lda, W, ldw, C, ldc, nullptr, 0, M, N, K, kStoreF32, st);
    return 1;
}

bool launch_gemm_swiglu(const bf16* A, int lda, const bf16* W13, int ldw, bf16* Hd, int ldh, int M,
                        int N, int K, cudaStream_t st) {
    if (!tc_gemm_enabled() || N % (2 * kW13Block)) return false;
    return launch_gemm_tc(A, lda, W13, ldw, nullptr, 0, Hd, ldh, M, N, K, kSwiGLU, 1, 0, st);
}

}  // namespace rlt
