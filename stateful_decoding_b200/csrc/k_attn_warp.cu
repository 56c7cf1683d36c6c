// Warp-per-(row, head) softmax attention for the three attention sites of
// RLT: the causal encoder (over the encoder cache C^E), the decoder's sliding
// window (over the ring cache C^D plus the block's own positions), and the
// decoder's cross-attention to the prefix memory M_{<=t} (jiphyeonjeon review
// §2-§3.3; greeksharifa §2.2, §2.5).
//
// Each warp runs an online softmax over its keys, 32 at a time: lane l scores
// key j0+l, the warp takes the block maximum and rescales, and every lane then
// accumulates its own output dimensions (lane, lane+32, ...) over the 32
// keys in order.  The summation order depends only on the key count, so the
// result of a row does not depend on the batch.
#include <math.h>

#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "kernels.cuh"

namespace rlt {

bool launch_attn_cross_fast(const float* Q, const bf16* mem, size_t row_stride, int T_cap,
                            const int32_t* pos_dec, bf16* A, int B, int n, int heads, int dh,
                            cudaStream_t st);
bool launch_attn_swa_fast(const float* Q, const bf16* Kc, const bf16* Vc, const bf16* ring,
                          size_t row_stride, int W, const int32_t* pos_dec, bf16* A, int B, int n,
                          int heads, int dh, cudaStream_t st);

// RLT_ATTN=warp keeps the decoder on the warp-per-head kernels (diagnostics)
bool fast_attn_enabled() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("RLT_ATTN");
        v = (e && strcmp(e, "warp") == 0) ? 0 : 1;
    }
    return v == 1;
}

namespace {

template <int DH> struct Nd { static constexpr int v = (DH + 31) / 32; };

template <typename T, int DH, typename KF, typename VF>
__device__ __forceinline__ void attend_range(const float* __restrict__ q, int nk, KF kf, VF vf,
                                             float& m, float& l, float (&acc)[Nd<DH>::v]) {
    const int lane = threadIdx.x & 31;
    for (int j0 = 0; j0 < nk; j0 += 32) {
        int j = j0 + lane;
        float s = -INFINITY;
        if (j < nk) {
            const T* kp = kf(j);
            float dot = 0.f;
#pragma unroll 16
            for (int x = 0; x < DH; ++x) dot = fmaf(q[x], to_f(kp[x]), dot);
            s = dot;
        }
        float mn = fmaxf(m, warp_max(s));
        float p = (j < nk) ? expf(s - mn) : 0.f;
        float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
        l = l * corr + warp_sum(p);
#pragma unroll
        for (int i = 0; i < Nd<DH>::v; ++i) acc[i] *= corr;
        int cnt = min(32, nk - j0);
        for (int jj = 0; jj < cnt; ++jj) {
            float pj = __shfl_sync(0xffffffffu, p, jj);
            const T* vp = vf(j0 + jj);
#pragma unroll
            for (int i = 0; i < Nd<DH>::v; ++i) {
                int dim = lane + 32 * i;
                if (dim < DH) acc[i] = fmaf(pj, to_f(vp[dim]), acc[i]);
            }
        }
        m = mn;
    }
}

template <typename T, int DH>
__device__ __forceinline__ void write_out(T* __restrict__ A, size_t off, float l,
                                          const float (&acc)[Nd<DH>::v]) {
    const int lane = threadIdx.x & 31;
    float inv = 1.0f / l;
#pragma unroll
    for (int i = 0; i < Nd<DH>::v; ++i) {
        int dim = lane + 32 * i;
        if (dim < DH) A[off + dim] = from_f<T>(acc[i] * inv);
    }
}

// Stage this warp's query (scaled by 1/sqrt(dh)) in shared memory.
template <int DH>
__device__ __forceinline__ float* stage_q(const float* __restrict__ Q, size_t off, float* sm) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float* q = sm + w * DH;
    const float sc = 1.0f / sqrtf((float)DH);
    for (int x = lane; x < DH; x += 32) q[x] = Q[off + x] * sc;
    __syncwarp();
    return q;
}

template <typename T, int DH>
__global__ void k_attn_enc(const float* __restrict__ Q, const T* __restrict__ cache,
                           size_t row_stride, int T_cap, const int32_t* __restrict__ pos_enc,
                           T* __restrict__ A, int R, int n, int heads) {
    pdl_enter();
    __shared__ float sm[4 * DH];
    int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (item >= R * heads) return;
    int r = item / heads, h = item % heads, b = r / n, i = r % n;
    int d = heads * DH;
    int t = pos_enc[b] + 1 + i;
    const float* q = stage_q<DH>(Q, (size_t)r * d + h * DH, sm);
    const T* kb = cache + (size_t)b * row_stride + (size_t)h * T_cap * DH;
    const T* vb = kb + (size_t)heads * T_cap * DH;
    float m = -INFINITY, l = 0.f, acc[Nd<DH>::v] = {};
    attend_range<T, DH>(q, t, [&](int j) { return kb + (size_t)j * DH; },
                        [&](int j) { return vb + (size_t)j * DH; }, m, l, acc);
    write_out<T, DH>(A, (size_t)r * d + h * DH, l, acc);
}

template <typename T, int DH>
__global__ void k_attn_swa(const float* __restrict__ Q, const T* __restrict__ Kc,
                           const T* __restrict__ Vc, const T* __restrict__ ring,
                           size_t row_stride, int W, const int32_t* __restrict__ pos_dec,
                           T* __restrict__ A, int R, int n, int heads) {
    pdl_enter();
    __shared__ float sm[4 * DH];
    int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (item >= R * heads) return;
    int r = item / heads, h = item % heads, b = r / n, i = r % n;
    int d = heads * DH;
    int pd = pos_dec[b];
    int t = pd + 1 + i;
    int nk = min(t, W);
    int p0 = t - nk + 1;                  // window t-W+1..t, clipped at 1
    int slots = W - 1;
    const float* q = stage_q<DH>(Q, (size_t)r * d + h * DH, sm);
    const T* rk = ring + (size_t)b * row_stride + (size_t)h * (slots > 0 ? slots : 1) * DH;
    const T* rv = rk + (size_t)heads * slots * DH;
    const T* ck = Kc + (size_t)b * n * d + h * DH;
    const T* cv = Vc + (size_t)b * n * d + h * DH;
    auto kf = [&](int j) {
        int p = p0 + j;
        return p <= pd ? rk + (size_t)((p - 1) % slots) * DH : ck + (size_t)(p - pd - 1) * d;
    };
    auto vf = [&](int j) {
        int p = p0 + j;
        return p <= pd ? rv + (size_t)((p - 1) % slots) * DH : cv + (size_t)(p - pd - 1) * d;
    };
    float m = -INFINITY, l = 0.f, acc[Nd<DH>::v] = {};
    attend_range<T, DH>(q, nk, kf, vf, m, l, acc);
    write_out<T, DH>(A, (size_t)r * d + h * DH, l, acc);
}

template <typename T, int DH>
__global__ void k_attn_cross(const float* __restrict__ Q, const T* __restrict__ mem,
                             size_t row_stride, int T_cap, const int32_t* __restrict__ pos_dec,
                             T* __restrict__ A, int R, int n, int heads) {
    pdl_enter();
    __shared__ float sm[4 * DH];
    int item = blockIdx.x * 4 + (threadIdx.x >> 5);
    if (item >= R * heads) return;
    int r = item / heads, h = item % heads, b = r / n, i = r % n;
    int d = heads * DH;
    int t = pos_dec[b] + 1 + i;
    const float* q = stage_q<DH>(Q, (size_t)r * d + h * DH, sm);
    const T* kb = mem + (size_t)b * row_stride + (size_t)h * T_cap * DH;
    const T* vb = kb + (size_t)heads * T_cap * DH;
    float m = -INFINITY, l = 0.f, acc[Nd<DH>::v] = {};
    attend_range<T, DH>(q, t, [&](int j) { return kb + (size_t)j * DH; },
                        [&](int j) { return vb + (size_t)j * DH; }, m, l, acc);
    write_out<T, DH>(A, (size_t)r * d + h * DH, l, acc);
}

inline int nblocks(int R, int heads) { return (R * heads + 3) / 4; }

}  // namespace

#define RLT_DH_SWITCH(dh, ...)                                     \
    switch (dh) {                                                  \
        case 16: { constexpr int DH = 16; __VA_ARGS__; } break;    \
        case 32: { constexpr int DH = 32; __VA_ARGS__; } break;    \
        case 64: { constexpr int DH = 64; __VA_ARGS__; } break;    \
        case 128: { constexpr int DH = 128; __VA_ARGS__; } break;  \
        default: return;                                           \
    }

template <typename T>
void launch_attn_enc(const float* Q, const T* cache, size_t row_stride, int T_cap,
                     const int32_t* pos_enc, T* A, int B, int n, int heads, int dh,
                     cudaStream_t st) {
    int R = B * n;
    if (R <= 0) return;
    // the encoder's causal attention is the same prefix read as the memory
    // read: queries at pos_enc+1+i over cache keys 1..t
    if constexpr (std::is_same<T, bf16>::value) {
        if (fast_attn_enabled() &&
            launch_attn_cross_fast(Q, cache, row_stride, T_cap, pos_enc, A, B, n, heads, dh, st))
            return;
    }
    RLT_DH_SWITCH(dh, (launch(k_attn_enc<T, DH>, nblocks(R, heads), 128, 0, st,
                          Q, cache, row_stride, T_cap, pos_enc, A, R, n, heads)));
    rlt_count_launch();
}

template <typename T>
void launch_attn_swa(const float* Q, const T* Kc, const T* Vc, const T* ring, size_t row_stride,
                     int W, const int32_t* pos_dec, T* A, int B, int n, int heads, int dh,
                     cudaStream_t st) {
    int R = B * n;
    if (R <= 0) return;
    if constexpr (std::is_same<T, bf16>::value) {
        if (fast_attn_enabled() &&
            launch_attn_swa_fast(Q, Kc, Vc, ring, row_stride, W, pos_dec, A, B, n, heads, dh, st))
            return;
    }
    RLT_DH_SWITCH(dh, (launch(k_attn_swa<T, DH>, nblocks(R, heads), 128, 0, st,
                          Q, Kc, Vc, ring, row_stride, W, pos_dec, A, R, n, heads)));
    rlt_count_launch();
}

template <typename T>
void launch_attn_cross(const float* Q, const T* mem, size_t row_stride, int T_cap,
                       const int32_t* pos_dec, T* A, int B, int n, int heads, int dh,
                       cudaStream_t st) {
    int R = B * n;
    if (R <= 0) return;
    if constexpr (std::is_same<T, bf16>::value) {
        if (fast_attn_enabled() &&
            launch_attn_cross_fast(Q, mem, row_stride, T_cap, pos_dec, A, B, n, heads, dh, st))
            return;
    }
    RLT_DH_SWITCH(dh, (launch(k_attn_cross<T, DH>, nblocks(R, heads), 128, 0, st,
                          Q, mem, row_stride, T_cap, pos_dec, A, R, n, heads)));
    rlt_count_launch();
}

#define RLT_INST(T)                                                                           \
    template void launch_attn_enc<T>(const float*, const T*, size_t, int, const int32_t*, T*, \
                                     int, int, int, int, cudaStream_t);                       \
    template void launch_attn_swa<T>(const float*, const T*, const T*, const T*, size_t, int, \
                                     const int32_t*, T*, int, int, int, int, cudaStream_t);   \
    template void launch_attn_cross<T>(const float*, const T*, size_t, int, const int32_t*,   \
                                       T*, int, int, int, int, cudaStream_t);
RLT_INST(float)
RLT_INST(bf16)
#undef RLT_INST

}  // namespace rlt
