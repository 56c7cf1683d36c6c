// Failure-detection self-test: a kernel whose one wait can never be
// satisfied, so that the bounded-wait path -- give up, record the timeout in
// the state's error word, return -- runs on the device on demand.  It uses
// the same helpers as the library's pipelines: tc::mbar_wait on an mbarrier
// (kind 0) and a polled word in global memory (kind 1, the form a grid
// barrier takes).  Nothing is in flight when a wait gives up (no bulk copy
// was issued, no TMEM is held), so the CTA may simply return.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace {

__device__ int g_never_set;      // no kernel ever writes it (zero-initialised)

__global__ void k_selftest_wait(int kind, uint32_t polls, int* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);           // one arrival expected; none will come
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    bool ok = false;
    if (kind == 0) {
        ok = tc::mbar_wait(&bar, 0, polls);
    } else {
        const volatile int* flag = &g_never_set;
        for (uint32_t i = 0; i < polls && !ok; ++i) {
            ok = *flag != 0;
            if (!ok) __nanosleep(256);
        }
    }
    if (!ok) atomicExch(err, kDevTimeout);
}

}  // namespace

void launch_selftest_wait(int kind, uint32_t polls, int* err, cudaStream_t st) {
    k_selftest_wait<<<1, 32, 0, st>>>(kind, polls, err);
    rlt_count_launch();
}

}  // namespace rlt
