// Readout tail: argmax and inverse-CDF sampling over the logits of each row
// (greeksharifa §2.3: norm, linear readout, softmax).  One block per row.
//
// argmax: largest logit, lowest index among equal maxima.
// sample: p_i = exp((l_i - max)/temperature); the first index i whose running
// sum (index order, fp64) exceeds u * total, u the SplitMix64 uniform of
// (seed, row, step).  The untruncated softmax is sampled: no top-k / top-p
// (jiphyeonjeon review §6.2).  Each thread owns a contiguous index range, so
// the sum order is fixed by V alone.
#include <math.h>

#include "kernels.cuh"

namespace rlt {

namespace {
constexpr int NT = 256;

__device__ __forceinline__ double sampler_uniform(uint64_t seed, uint64_t row, uint64_t step) {
    uint64_t key = mix64(seed ^ mix64((row + 1) * kGolden));
    uint64_t x = mix64(key + (step + 1) * kGolden);
    return (double)(x >> 11) * (1.0 / 9007199254740992.0);
}

__global__ void __launch_bounds__(NT)
k_sample(const float* __restrict__ logits, int V, int32_t* __restrict__ argmax_out,
         int32_t* __restrict__ sampled_out, uint64_t seed, uint64_t step, float temperature) {
    pdl_enter();
    __shared__ float s_val[NT];
    __shared__ int s_idx[NT];
    __shared__ double s_sum[NT];
    __shared__ double s_excl[NT + 1];
    const int row = blockIdx.x, tid = threadIdx.x;
    const float* lg = logits + (size_t)row * V;
    const int chunk = (V + NT - 1) / NT;
    const int lo = min(V, tid * chunk), hi = min(V, lo + chunk);

    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lo; i < hi; ++i) {
        float v = lg[i];
        if (v > bv) { bv = v; bi = i; }
    }
    s_val[tid] = bv;
    s_idx[tid] = bi;
    __syncthreads();
    for (int off = NT / 2; off > 0; off >>= 1) {
        if (tid < off) {
            float v2 = s_val[tid + off];
            int i2 = s_idx[tid + off];
            if (v2 > s_val[tid] || (v2 == s_val[tid] && i2 < s_idx[tid])) {
                s_val[tid] = v2;
                s_idx[tid] = i2;
            }
        }
        __syncthreads();
    }
    const float mx = s_val[0];
    const int amax = s_idx[0];
    if (tid == 0 && argmax_out) argmax_out[row] = amax;
    if (!sampled_out) return;

    const float inv_t = 1.0f / temperature;
    double local = 0.0;
    for (int i = lo; i < hi; ++i) local += (double)expf((lg[i] - mx) * inv_t);
    s_sum[tid] = local;
    __syncthreads();
    if (tid == 0) {
        double acc = 0.0;
        for (int k = 0; k < NT; ++k) {
            s_excl[k] = acc;
            acc += s_sum[k];
        }
        s_excl[NT] = acc;
    }
    __syncthreads();
    const double total = s_excl[NT];
    const double target = sampler_uniform(seed, (uint64_t)row, step) * total;
    if (target >= s_excl[tid] && target < s_excl[tid] + s_sum[tid] && hi > lo) {
        // same additions from 0 as `local`, so the last partial sum is `local`
        // and some index of the range satisfies the test
        double run = 0.0;
        int pick = hi - 1;
        for (int i = lo; i < hi; ++i) {
            run += (double)expf((lg[i] - mx) * inv_t);
            if (s_excl[tid] + run > target) { pick = i; break; }
        }
        sampled_out[row] = pick;
    }
    if (tid == 0 && !(target < total)) {
        // u * total rounded up to the total: the last index with p > 0
        int pick = V - 1;
        for (int i = V - 1; i >= 0; --i)
            if (expf((lg[i] - mx) * inv_t) > 0.f) { pick = i; break; }
        sampled_out[row] = pick;
    }
}

// log softmax(logits / temperature)[id] for one given id per row: the log of
// the probability k_sample draws that id with, its max and its fp64 sum
// formed the same way (each thread a contiguous index range, the partial sums
// added in thread order).  This is the per-token term of the policy's
// log-likelihood that a replay reads before consuming the token
// (jiphyeonjeon review §6.2, eq. 5.3 and 5.5).  An id outside [0, V) gives
// NaN and the bounds code in *err.
__global__ void __launch_bounds__(NT)
k_logprob(const float* __restrict__ logits, int V, const int32_t* __restrict__ ids,
          int ids_stride, float* __restrict__ out, int out_stride, float temperature,
          int* __restrict__ err) {
    pdl_enter();
    __shared__ float s_max[NT];
    __shared__ double s_sum[NT];
    const int row = blockIdx.x, tid = threadIdx.x;
    const float* lg = logits + (size_t)row * V;
    const int chunk = (V + NT - 1) / NT;
    const int lo = min(V, tid * chunk), hi = min(V, lo + chunk);

    float bv = -INFINITY;
    for (int i = lo; i < hi; ++i) bv = fmaxf(bv, lg[i]);
    s_max[tid] = bv;
    __syncthreads();
    for (int off = NT / 2; off > 0; off >>= 1) {
        if (tid < off) s_max[tid] = fmaxf(s_max[tid], s_max[tid + off]);
        __syncthreads();
    }
    const float mx = s_max[0];
    const float inv_t = 1.0f / temperature;
    double local = 0.0;
    for (int i = lo; i < hi; ++i) local += (double)expf((lg[i] - mx) * inv_t);
    s_sum[tid] = local;
    __syncthreads();
    if (tid == 0) {
        double total = 0.0;
        for (int k = 0; k < NT; ++k) total += s_sum[k];
        const int id = ids[(size_t)row * ids_stride];
        float lp = NAN;
        if (id >= 0 && id < V)
            lp = (float)((double)((lg[id] - mx) * inv_t) - log(total));
        else if (err)
            atomicExch(err, kDevBounds);
        out[(size_t)row * out_stride] = lp;
    }
}
}  // namespace

void launch_logprob(const float* logits, int V, int B, const int32_t* ids, int ids_stride,
                    float* out, int out_stride, float temperature, int* err, cudaStream_t st) {
    if (B <= 0) return;
    launch(k_logprob, B, NT, 0, st, logits, V, ids, ids_stride, out, out_stride, temperature,
           err);
    rlt_count_launch();
}

void launch_sample(const float* logits, int V, int B, int32_t* argmax, int32_t* sampled,
                   uint64_t seed, uint64_t step, float temperature, cudaStream_t st) {
    if (B <= 0 || (!argmax && !sampled)) return;
    launch(k_sample, B, NT, 0, st, logits, V, argmax, sampled, seed, step, temperature);
    rlt_count_launch();
}

}  // namespace rlt
