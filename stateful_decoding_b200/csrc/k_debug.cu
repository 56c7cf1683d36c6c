// Debug-build validation of the per-row position counters (compiled in every
// build, launched only when RLT_DEBUG=1): before a transition block of n
// positions every row must have 0 <= pos_dec, pos_dec + n <= pos_enc and
// pos_enc <= T_cap; before an encoder block of n positions, pos_enc + n <=
// T_cap.  A violation records kDevOrder or kDevCapacity in the state's error
// word (the first code wins); nothing traps and nothing is modified.
#include "kernels.cuh"

namespace rlt {
namespace {

__global__ void k_check_positions(const int32_t* __restrict__ pos_enc,
                                  const int32_t* __restrict__ pos_dec, int B, int n, int T_cap,
                                  int encoding, int* err) {
    pdl_enter();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
        const int pe = __ldcg(pos_enc + b), pd = __ldcg(pos_dec + b);
        if (encoding) {
            if (pe < 0 || pe + n > T_cap) atomicCAS(err, 0, kDevCapacity);
        } else {
            if (pe > T_cap || pd < 0) atomicCAS(err, 0, kDevCapacity);
            else if (pd + n > pe) atomicCAS(err, 0, kDevOrder);
        }
    }
}

}  // namespace

void launch_check_positions(const int32_t* pos_enc, const int32_t* pos_dec, int B, int n,
                            int T_cap, bool encoding, int* err, cudaStream_t st) {
    if (!RLT_DEBUG || B <= 0) return;
    launch(k_check_positions, (B + 255) / 256, 256, 0, st, pos_enc, pos_dec, B, n, T_cap,
           encoding ? 1 : 0, err);
    rlt_count_launch();
}

}  // namespace rlt
