// Device helpers shared by the RLT kernels: storage types, warp reductions,
// the SplitMix64 finaliser, and the launch bookkeeping the C ABI exposes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace rlt {

typedef __nv_bfloat16 bf16;

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// SplitMix64 output function (Steele, Lea, Flood 2014).
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
static constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

// Sticky per-state error codes written by device code (0 = none).
enum DevError : int {
    kDevOk = 0,
    kDevTimeout = 1,     // a bounded wait gave up
    kDevBounds = 2,      // a token id outside [0, vocab)
    kDevOrder = 3,       // debug builds: a block would consume positions not yet encoded
    kDevCapacity = 4,    // debug builds: a position or ring slot outside its buffer
};

// RLT_DEBUG=1 (the librlt_debug.so build) compiles in bounds checks of
// positions, ring slots and key indices; a failed check records its code in
// the error word (the first code wins) and the access it guards is skipped.
// Nothing traps.
#ifndef RLT_DEBUG
#define RLT_DEBUG 0
#endif
__device__ __forceinline__ bool dcheck(bool ok, int* err, int code) {
#if RLT_DEBUG
    if (!ok) atomicCAS(err, 0, code);
    return ok;
#else
    (void)err;
    (void)code;
    return true;
#endif
}

}  // namespace rlt

// Launch bookkeeping (defined in rlt_api.cu).
void rlt_count_launch(int n = 1);

// Programmatic dependent launch.  Every kernel of the library starts with
// pdl_wait() (before it reads or writes anything an earlier kernel of the
// stream touches) and then lets the next kernel of the stream begin its own
// launch and prologue.  Both are no-ops in a kernel launched without the
// attribute.
namespace rlt {
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
    pdl_wait();
    pdl_trigger();
}

// True unless RLT_PDL=0 (defined in rlt_api.cu).
bool pdl_enabled();
// Once per kernel: the same preferred shared-memory carveout (all shared)
// for every kernel of the library, so that consecutive kernels never make an
// SM switch its L1 / shared-memory split (defined in rlt_api.cu).
void set_carveout_once(const void* kernel);
// The kernel's dynamic shared-memory limit, set once per (device, kernel,
// size); false when the device refuses it.
bool set_smem_once(const void* kernel, size_t bytes);
// Multiprocessors of the current device (0 on error).
int sm_count();

// kernel<<<grid, block, smem, st>>>(args...) with the programmatic-serialisation
// attribute set when PDL is enabled.
template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    set_carveout_once(reinterpret_cast<const void*>(kernel));
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
}  // namespace rlt
