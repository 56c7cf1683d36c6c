// Row-wise kernels of the RLT path: embedding, RMSNorm, the merge gate
// (greeksharifa "Recurrent Looped Transformer 요약 설명" §2.5), RoPE scatters
// into the encoder cache / memory / window chunk, SwiGLU, state hand-off and
// the window-cache (ring) update of jiphyeonjeon review §3.3.
#include <algorithm>

#include "kernels.cuh"

namespace rlt {

// Sum of S split-K partial slabs (slab z at P + z*slab), in slab order.
__device__ __forceinline__ float slab_sum(const float* __restrict__ P, int S, size_t slab,
                                          size_t i) {
    float v = P[i];
    for (int z = 1; z < S; ++z) v += P[(size_t)z * slab + i];
    return v;
}

// ---------------------------------------------------------------- row kernels
// The decoder's row kernels give each thread one group of 4 consecutive
// features (blockDim = d/4 rounded up to a warp), so that every load a thread
// needs -- the row and each split-K partial slab -- is issued before the
// first is used: one memory latency per kernel instead of a chain of them.
constexpr int kMaxSlabs = 8;       // split-K slabs a consumer sums (the splitter caps at this)

__device__ __forceinline__ float4 ld4(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float dot4(float4 a) { return a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w; }
// sum of S partial slabs at element i (4 wide), in slab order
__device__ __forceinline__ float4 slab_sum4(const float* __restrict__ P, int S, size_t slab,
                                            size_t i) {
    float4 t[kMaxSlabs];
#pragma unroll
    for (int z = 0; z < kMaxSlabs; ++z)
        if (z < S) t[z] = ld4(P + (size_t)z * slab + i);
    float4 v = t[0];
#pragma unroll
    for (int z = 1; z < kMaxSlabs; ++z)
        if (z < S) v = add4(v, t[z]);
    return v;
}
template <typename T> __device__ __forceinline__ void store4(T* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) { st4(p, v); }
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}
// Block-wide sum with a fixed order (warp butterfly, then the warp partials
// in warp order, summed by every thread alike).
__device__ __forceinline__ float row_sum(float v, float* red) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
    for (int i = 0; i < nw; ++i) s += red[i];
    return s;
}
__host__ __forceinline__ int row_threads(int groups) { return ((groups + 31) / 32) * 32; }
__device__ __forceinline__ float4 scale4(float4 v, float inv, float4 g) {
    return make_float4(v.x * inv * g.x, v.y * inv * g.y, v.z * inv * g.z, v.w * inv * g.w);
}

// ---------------------------------------------------------------- embedding
template <typename T>
__global__ void k_embed(const T* __restrict__ E, const int32_t* __restrict__ tok,
                        float* __restrict__ X, int d, int vocab, int* err) {
    pdl_enter();
    int r = blockIdx.x;
    int id = tok[r];
    bool ok = id >= 0 && id < vocab;
    if (!ok && threadIdx.x == 0 && err) atomicExch(err, kDevBounds);
    for (int j = threadIdx.x; j < d; j += blockDim.x)
        X[(size_t)r * d + j] = ok ? to_f(E[(size_t)id * d + j]) : 0.f;
}
template <typename T>
void launch_embed(const T* E, const int32_t* tok, float* X, int R, int d, int vocab, int* err,
                  cudaStream_t st) {
    if (R <= 0) return;
    launch(k_embed<T>, R, 128, 0, st, E, tok, X, d, vocab, err);
    rlt_count_launch();
}

// ---------------------------------------------------------------- RMSNorm
// One warp per row (d <= 2048: at most 16 float4 groups per lane), 8 rows
// per block; the row is loaded once, squares summed per lane then across
// the warp in a fixed order.
template <typename T>
__global__ void __launch_bounds__(256) k_rmsnorm(const float* __restrict__ X, int ldx,
                                                 const float* __restrict__ g, T* __restrict__ Y,
                                                 int ldy, int R, int d, float eps) {
    pdl_enter();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= R) return;
    const float* x = X + (size_t)row * ldx;
    const int d4 = d / 4;
    float4 v[16];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const int j4 = lane + 32 * c;
        if (j4 < d4) {
            v[c] = ld4(x + 4 * j4);
            ss += dot4(v[c]);
        }
    }
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    T* y = Y + (size_t)row * ldy;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const int j4 = lane + 32 * c;
        if (j4 < d4) store4<T>(y + 4 * j4, scale4(v[c], inv, ld4(g + 4 * j4)));
    }
}
template <typename T>
void launch_rmsnorm(const float* X, int ldx, const float* gain, T* Y, int ldy, int R, int d,
                    float eps, cudaStream_t st) {
    if (R <= 0) return;
    launch(k_rmsnorm<T>, (R + 7) / 8, 256, 0, st, X, ldx, gain, Y, ldy, R, d, eps);
    rlt_count_launch();
}

// z += sum of the residual partial slabs P (if any), then Y = RMSNorm(z).
template <typename T>
__global__ void __launch_bounds__(512) k_add_rmsnorm(float* __restrict__ Z, const float* __restrict__ P, int S,
                              size_t slab, const float* __restrict__ g, T* __restrict__ Y, int d,
                              float eps) {
    pdl_enter();
    __shared__ float red[32];
    const int j = 4 * threadIdx.x;
    const size_t i = (size_t)blockIdx.x * d + j;
    const bool act = j < d;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f), gv = v;
    if (act) {
        gv = ld4(g + j);
        v = ld4(Z + i);
        if (P) {
            v = add4(v, slab_sum4(P, S, slab, i));
            st4(Z + i, v);
        }
    }
    const float ss = row_sum(act ? dot4(v) : 0.f, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    if (act) store4<T>(Y + i, scale4(v, inv, gv));
}
template <typename T>
void launch_add_rmsnorm(float* Z, const float* P, int S, size_t slab, const float* gain, T* Y,
                        int R, int d, float eps, cudaStream_t st) {
    if (R <= 0) return;
    launch(k_add_rmsnorm<T>, R, row_threads(d / 4), 0, st, Z, P, S, slab, gain, Y, d, eps);
    rlt_count_launch();
}

// ---------------------------------------------------------------- merge
template <typename T>
__global__ void __launch_bounds__(512) k_merge_input(const float* __restrict__ e, int T_cap,
                              const int32_t* __restrict__ pos_dec, const float* __restrict__ fb,
                              const float* __restrict__ g, T* __restrict__ Gin, int n, int d,
                              float eps) {
    pdl_enter();
    __shared__ float red[32];
    const int r = blockIdx.x, b = r / n, i = r % n;
    const int j = 4 * threadIdx.x;
    const bool act = j < d;
    float4 ev = make_float4(0.f, 0.f, 0.f, 0.f), f = ev, gv = ev;
    if (act) {
        ev = ld4(e + ((size_t)b * T_cap + pos_dec[b] + i) * d + j);
        f = ld4(fb + (size_t)b * d + j);
        gv = ld4(g + j);
    }
    const float ss = row_sum(act ? dot4(f) : 0.f, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    if (act) {
        T* out = Gin + (size_t)r * 2 * d;
        store4<T>(out + j, ev);
        store4<T>(out + d + j, scale4(f, inv, gv));
    }
}
template <typename T>
void launch_merge_input(const float* e, int T_cap, const int32_t* pos_dec, const float* fb,
                        const float* gain, T* Gin, int B, int n, int d, float eps,
                        cudaStream_t st) {
    launch(k_merge_input<T>, B * n, row_threads(d / 4), 0, st, e, T_cap, pos_dec, fb, gain, Gin,
           n, d, eps);
    rlt_count_launch();
}

// z = e_t + alpha * sigma(gate) * projection; with a gain, also Y = RMSNorm(z)
// (the first decoder block's input norm, same arithmetic as k_add_rmsnorm).
template <typename T>
__global__ void __launch_bounds__(512) k_merge_out(const float* __restrict__ e, int T_cap,
                            const int32_t* __restrict__ pos_dec, const float* __restrict__ G,
                            int nG, size_t slabG, const float* __restrict__ bg,
                            const float* __restrict__ S, int nS, size_t slabS, int ldg,
                            float alpha, float* __restrict__ z, int n, int d,
                            const float* __restrict__ g, T* __restrict__ Y, float eps) {
    pdl_enter();
    __shared__ float red[32];
    const int r = blockIdx.x, b = r / n, i = r % n;
    const int j = 4 * threadIdx.x;
    const bool act = j < d;
    const size_t o = (size_t)r * d + j;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f), gv = u;
    if (act) {
        u = ld4(e + ((size_t)b * T_cap + pos_dec[b] + i) * d + j);
        if (g) gv = ld4(g + j);
        if (G) {
            const size_t og = (size_t)r * ldg + j;      // G and S rows have pitch ldg
            const float4 a = add4(slab_sum4(G, nG, slabG, og), ld4(bg + j));
            const float4 p = slab_sum4(S, nS, slabS, og);
            u.x += alpha * (1.0f / (1.0f + expf(-a.x))) * p.x;
            u.y += alpha * (1.0f / (1.0f + expf(-a.y))) * p.y;
            u.z += alpha * (1.0f / (1.0f + expf(-a.z))) * p.z;
            u.w += alpha * (1.0f / (1.0f + expf(-a.w))) * p.w;
        }
        st4(z + o, u);
    }
    if (!g) return;
    const float ss = row_sum(act ? dot4(u) : 0.f, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    if (act) store4<T>(Y + o, scale4(u, inv, gv));
}
template <typename T>
void launch_merge_out(const float* e, int T_cap, const int32_t* pos_dec, const float* G, int nG,
                      size_t slabG, const float* bg, const float* S, int nS, size_t slabS,
                      int ldg, float alpha, float* z, const float* gain, T* Y, float eps, int B,
                      int n, int d, cudaStream_t st) {
    launch(k_merge_out<T>, B * n, row_threads(d / 4), 0, st, e, T_cap, pos_dec, G, nG, slabG, bg,
           S, nS, slabS, ldg, alpha, z, n, d, gain, Y, eps);
    rlt_count_launch();
}

// ---------------------------------------------------------------- RoPE scatters
// rotate-half: pair (j, j+half) turns by p * base^(-2j/dh) (rope_pair)

template <typename T>
__global__ void k_qkv_dec(const float* __restrict__ QKV, int S, size_t slab,
                          const int32_t* __restrict__ pos_dec, RopeTab rope,
                          float* __restrict__ Q, T* __restrict__ Kc, T* __restrict__ Vc, int n,
                          int heads, int dh) {
    pdl_enter();
    int r = blockIdx.x, b = r / n, i = r % n;
    int d = heads * dh, half = dh / 2;
    int t = pos_dec[b] + 1 + i;
    const size_t base = (size_t)r * 3 * d;
    for (int x = threadIdx.x; x < heads * half; x += blockDim.x) {
        int h = x / half, j = x % half;
        float c = rope.cs[(size_t)t * half + j], s = rope.sn[(size_t)t * half + j];
        int o1 = h * dh + j, o2 = o1 + half;
        float y1, y2;
        rope_pair(slab_sum(QKV, S, slab, base + o1), slab_sum(QKV, S, slab, base + o2), c, s, y1, y2);
        Q[(size_t)r * d + o1] = y1;
        Q[(size_t)r * d + o2] = y2;
        rope_pair(slab_sum(QKV, S, slab, base + d + o1), slab_sum(QKV, S, slab, base + d + o2), c, s, y1,
            y2);
        Kc[(size_t)r * d + o1] = from_f<T>(y1);
        Kc[(size_t)r * d + o2] = from_f<T>(y2);
        Vc[(size_t)r * d + o1] = from_f<T>(slab_sum(QKV, S, slab, base + 2 * d + o1));
        Vc[(size_t)r * d + o2] = from_f<T>(slab_sum(QKV, S, slab, base + 2 * d + o2));
    }
}
template <typename T>
void launch_qkv_dec(const float* QKV, int S, size_t slab, const int32_t* pos_dec, RopeTab rope,
                    float* Q, T* Kc, T* Vc, int B, int n, int heads, int dh, cudaStream_t st) {
    launch(k_qkv_dec<T>, B * n, 128, 0, st, QKV, S, slab, pos_dec, rope, Q, Kc, Vc, n, heads, dh);
    rlt_count_launch();
}

// cache layout per sequence: [2][heads][T_cap][dh] starting at cache + b*row_stride
template <typename T>
__global__ void k_qkv_enc(const float* __restrict__ QKV, const int32_t* __restrict__ pos_enc,
                          RopeTab rope, float* __restrict__ Q, T* __restrict__ cache,
                          size_t row_stride, int T_cap, int n, int heads, int dh) {
    pdl_enter();
    int r = blockIdx.x, b = r / n, i = r % n;
    int d = heads * dh, half = dh / 2;
    int p = pos_enc[b] + 1 + i;
    const float* src = QKV + (size_t)r * 3 * d;
    T* kc = cache + (size_t)b * row_stride;
    T* vc = kc + (size_t)heads * T_cap * dh;
    for (int x = threadIdx.x; x < heads * half; x += blockDim.x) {
        int h = x / half, j = x % half;
        float c = rope.cs[(size_t)p * half + j], s = rope.sn[(size_t)p * half + j];
        int o1 = h * dh + j, o2 = o1 + half;
        size_t dst = ((size_t)h * T_cap + (p - 1)) * dh + j;
        float y1, y2;
        rope_pair(src[o1], src[o2], c, s, y1, y2);
        Q[(size_t)r * d + o1] = y1;
        Q[(size_t)r * d + o2] = y2;
        rope_pair(src[d + o1], src[d + o2], c, s, y1, y2);
        kc[dst] = from_f<T>(y1);
        kc[dst + half] = from_f<T>(y2);
        vc[dst] = from_f<T>(src[2 * d + o1]);
        vc[dst + half] = from_f<T>(src[2 * d + o2]);
    }
}
template <typename T>
void launch_qkv_enc(const float* QKV, const int32_t* pos_enc, RopeTab rope, float* Q, T* cache,
                    size_t row_stride, int T_cap, int B, int n, int heads, int dh,
                    cudaStream_t st) {
    launch(k_qkv_enc<T>, B * n, 128, 0, st, QKV, pos_enc, rope, Q, cache, row_stride, T_cap, n,
                                        heads, dh);
    rlt_count_launch();
}

template <typename T>
__global__ void k_mem_scatter(const float* __restrict__ KV, const int32_t* __restrict__ pos_enc,
                              RopeTab rope, T* __restrict__ mem, size_t row_stride, int T_cap,
                              int n, int heads, int dh) {
    pdl_enter();
    int r = blockIdx.x, b = r / n, i = r % n;
    int d = heads * dh, half = dh / 2;
    int p = pos_enc[b] + 1 + i;
    const float* src = KV + (size_t)r * 2 * d;
    T* mk = mem + (size_t)b * row_stride;
    T* mv = mk + (size_t)heads * T_cap * dh;
    for (int x = threadIdx.x; x < heads * half; x += blockDim.x) {
        int h = x / half, j = x % half;
        float c = rope.cs[(size_t)p * half + j], s = rope.sn[(size_t)p * half + j];
        int o1 = h * dh + j, o2 = o1 + half;
        size_t dst = ((size_t)h * T_cap + (p - 1)) * dh + j;
        float y1, y2;
        rope_pair(src[o1], src[o2], c, s, y1, y2);
        mk[dst] = from_f<T>(y1);
        mk[dst + half] = from_f<T>(y2);
        mv[dst] = from_f<T>(src[d + o1]);
        mv[dst + half] = from_f<T>(src[d + o2]);
    }
}
template <typename T>
void launch_mem_scatter(const float* KV, const int32_t* pos_enc, RopeTab rope, T* mem,
                        size_t row_stride, int T_cap, int B, int n, int heads, int dh,
                        cudaStream_t st) {
    launch(k_mem_scatter<T>, B * n, 128, 0, st, KV, pos_enc, rope, mem, row_stride, T_cap, n, heads,
                                            dh);
    rlt_count_launch();
}

__global__ void k_rope_q(const float* __restrict__ P, int S, size_t slab,
                         float* __restrict__ Q, const int32_t* __restrict__ pos_dec,
                         RopeTab rope, int n, int heads, int dh) {
    pdl_enter();
    int r = blockIdx.x, b = r / n, i = r % n;
    int d = heads * dh, half = dh / 2;
    int t = pos_dec[b] + 1 + i;
    for (int x = threadIdx.x; x < heads * half; x += blockDim.x) {
        int h = x / half, j = x % half;
        float c = rope.cs[(size_t)t * half + j], s = rope.sn[(size_t)t * half + j];
        int o1 = h * dh + j, o2 = o1 + half;
        float y1, y2;
        rope_pair(slab_sum(P, S, slab, (size_t)r * d + o1), slab_sum(P, S, slab, (size_t)r * d + o2), c,
            s, y1, y2);
        Q[(size_t)r * d + o1] = y1;
        Q[(size_t)r * d + o2] = y2;
    }
}
void launch_rope_q(const float* P, int S, size_t slab, float* Q, const int32_t* pos_dec,
                   RopeTab rope, int B, int n, int heads, int dh, cudaStream_t st) {
    launch(k_rope_q, B * n, 128, 0, st, P, S, slab, Q, pos_dec, rope, n, heads, dh);
    rlt_count_launch();
}

// ---------------------------------------------------------------- FFN gate
// grid (rows, ceil(fpad/4 / 256)): one group of 4 hidden units per thread
template <typename T>
__global__ void __launch_bounds__(256) k_swiglu(const float* __restrict__ H, int S, size_t slab,
                                                int fpad, T* __restrict__ Hd) {
    pdl_enter();
    const int r = blockIdx.x;
    const int j = 4 * (blockIdx.y * blockDim.x + threadIdx.x);
    if (j >= fpad) return;
    // interleaved W1;W3 (w13_gate_col): 4 consecutive units share a block
    const size_t base = (size_t)r * 2 * fpad + w13_gate_col(j);
    const float4 a = slab_sum4(H, S, slab, base);
    const float4 u = slab_sum4(H, S, slab, base + kW13Block);
    float4 y;
    y.x = silu_mul(a.x, u.x);
    y.y = silu_mul(a.y, u.y);
    y.z = silu_mul(a.z, u.z);
    y.w = silu_mul(a.w, u.w);
    store4<T>(Hd + (size_t)r * fpad + j, y);
}
template <typename T>
void launch_swiglu(const float* H, int S, size_t slab, int fpad, T* Hd, int R, cudaStream_t st) {
    if (R <= 0) return;
    launch(k_swiglu<T>, dim3(R, (fpad / 4 + 255) / 256), 256, 0, st, H, S, slab, fpad, Hd);
    rlt_count_launch();
}

// ---------------------------------------------------------------- state bookkeeping
__global__ void k_copy_e(const float* __restrict__ X, const int32_t* __restrict__ pos_enc,
                         float* __restrict__ e, int T_cap, int n, int d) {
    pdl_enter();
    int r = blockIdx.x, b = r / n, i = r % n;
    float* dst = e + ((size_t)b * T_cap + pos_enc[b] + i) * d;
    for (int j = threadIdx.x; j < d; j += blockDim.x) dst[j] = X[(size_t)r * d + j];
}
void launch_copy_e(const float* X, const int32_t* pos_enc, float* e, int T_cap, int B, int n,
                   int d, cudaStream_t st) {
    launch(k_copy_e, B * n, 128, 0, st, X, pos_enc, e, T_cap, n, d);
    rlt_count_launch();
}

// s <- last row of z (+ residual slabs); RLT-2 register when the chunk ends;
// with `bump`, also pos_dec += n once every thread has read it.
__global__ void __launch_bounds__(512) k_set_state(const float* __restrict__ z, const float* __restrict__ P, int S,
                            size_t slab, float* __restrict__ s, float* __restrict__ Rr,
                            int32_t* __restrict__ pos_dec, int chunk, int n, int d, int bump) {
    pdl_enter();
    const int b = blockIdx.x;
    const bool upd = Rr != nullptr && ((pos_dec[b] + n) % chunk) == 0;
    const int j = 4 * threadIdx.x;
    if (j < d) {
        const size_t row = ((size_t)b * n + n - 1) * d;
        float4 v = ld4(z + row + j);
        if (P) v = add4(v, slab_sum4(P, S, slab, row + j));
        st4(s + (size_t)b * d + j, v);
        if (upd) st4(Rr + (size_t)b * d + j, v);
    }
    if (bump) {
        __syncthreads();
        if (threadIdx.x == 0) pos_dec[b] += n;
    }
}
void launch_set_state(const float* z, const float* P, int S, size_t slab, float* s, float* Rreg,
                      int32_t* pos_dec, int chunk, int B, int n, int d, bool bump,
                      cudaStream_t st) {
    launch(k_set_state, B, row_threads(d / 4), 0, st, z, P, S, slab, s, Rreg, pos_dec, chunk, n, d,
           (int)bump);
    rlt_count_launch();
}

// One position per row: the state hand-off of this transition and the
// merge input of the next, in one kernel (rows of a replayed run of blocks):
// s <- z (+ residual slabs), RLT-2 register at a chunk end, pos_dec += 1, then
// Gin = [T(e at the new position), T(RMSNorm(s or R) * gain)].  Same
// arithmetic as k_set_state followed by k_merge_input.
template <typename T>
__global__ void __launch_bounds__(512)
k_state_merge(const float* __restrict__ z, const float* __restrict__ P, int S, size_t slab,
              float* __restrict__ s, float* __restrict__ Rr, int32_t* __restrict__ pos_dec,
              int chunk, const float* __restrict__ e, int T_cap, const float* __restrict__ g,
              T* __restrict__ Gin, int d, float eps) {
    pdl_enter();
    __shared__ float red[32];
    const int b = blockIdx.x;
    const int pd = pos_dec[b];
    const bool upd = Rr != nullptr && ((pd + 1) % chunk) == 0;
    const int j = 4 * threadIdx.x;
    const bool act = j < d;
    float4 fb = make_float4(0.f, 0.f, 0.f, 0.f), ev = fb, gv = fb;
    if (act) {
        const size_t row = (size_t)b * d + j;
        float4 v = ld4(z + row);
        if (P) v = add4(v, slab_sum4(P, S, slab, row));
        st4(s + row, v);
        fb = v;
        if (Rr) {
            if (upd) st4(Rr + row, v);
            else fb = ld4(Rr + row);
        }
        ev = ld4(e + ((size_t)b * T_cap + pd + 1) * d + j);
        gv = ld4(g + j);
    }
    const float ss = row_sum(act ? dot4(fb) : 0.f, red);   // every thread read pd before this
    if (threadIdx.x == 0) pos_dec[b] = pd + 1;
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    if (act) {
        T* out = Gin + (size_t)b * 2 * d;
        store4<T>(out + j, ev);
        store4<T>(out + d + j, scale4(fb, inv, gv));
    }
}
template <typename T>
void launch_state_merge(const float* z, const float* P, int S, size_t slab, float* s, float* Rreg,
                        int32_t* pos_dec, int chunk, const float* e, int T_cap, const float* gain,
                        T* Gin, int B, int d, float eps, cudaStream_t st) {
    launch(k_state_merge<T>, B, row_threads(d / 4), 0, st, z, P, S, slab, s, Rreg, pos_dec, chunk,
           e, T_cap, gain, Gin, d, eps);
    rlt_count_launch();
}

__global__ void k_pos_add(int32_t* pos, int B, int n) {
    pdl_enter();
    int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) pos[b] += n;
}
void launch_pos_add(int32_t* pos, int B, int n, cudaStream_t st) {
    launch(k_pos_add, (B + 255) / 256, 256, 0, st, pos, B, n);
    rlt_count_launch();
}

__global__ void k_reset_rows(const int32_t* __restrict__ rows, const float* __restrict__ s_star,
                             float* __restrict__ s, float* __restrict__ Rr,
                             int32_t* __restrict__ pos_enc, int32_t* __restrict__ pos_dec,
                             int d) {
    pdl_enter();
    int b = rows ? rows[blockIdx.x] : blockIdx.x;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        float v = s_star ? s_star[j] : 0.f;
        s[(size_t)b * d + j] = v;
        Rr[(size_t)b * d + j] = v;
    }
    if (threadIdx.x == 0) {
        pos_enc[b] = 0;
        pos_dec[b] = 0;
    }
}
void launch_reset_rows(const int32_t* rows, int nrows, const float* s_star, float* s, float* Rr,
                       int32_t* pos_enc, int32_t* pos_dec, int d, cudaStream_t st) {
    if (nrows <= 0) return;
    launch(k_reset_rows, nrows, 128, 0, st, rows, s_star, s, Rr, pos_enc, pos_dec, d);
    rlt_count_launch();
}

// ring layout per sequence and layer: [2][heads][W-1][dh]; position p lives in
// slot (p-1) mod (W-1).  Only the last W-1 positions of a block are written,
// so no two threads of one launch write the same slot.
template <typename T>
__global__ void k_ring_write(const T* __restrict__ Kc, const T* __restrict__ Vc,
                             const int32_t* __restrict__ pos_dec, T* __restrict__ ring,
                             size_t row_stride, int W, int n, int heads, int dh) {
    pdl_enter();
    int r = blockIdx.x, b = r / n, i = r % n;
    int slots = W - 1;
    if (i < n - slots) return;
    int p = pos_dec[b] + 1 + i;
    int slot = (p - 1) % slots;
    int d = heads * dh;
    T* rk = ring + (size_t)b * row_stride;
    T* rv = rk + (size_t)heads * slots * dh;
    for (int x = threadIdx.x; x < d; x += blockDim.x) {
        int h = x / dh, j = x % dh;
        size_t dst = ((size_t)h * slots + slot) * dh + j;
        rk[dst] = Kc[(size_t)r * d + x];
        rv[dst] = Vc[(size_t)r * d + x];
    }
}
template <typename T>
void launch_ring_write(const T* Kc, const T* Vc, const int32_t* pos_dec, T* ring,
                       size_t row_stride, int W, int B, int n, int heads, int dh,
                       cudaStream_t st) {
    if (W <= 1) return;
    launch(k_ring_write<T>, B * n, 128, 0, st, Kc, Vc, pos_dec, ring, row_stride, W, n, heads, dh);
    rlt_count_launch();
}

#define RLT_INST(T)                                                                            \
    template void launch_embed<T>(const T*, const int32_t*, float*, int, int, int, int*,       \
                                  cudaStream_t);                                               \
    template void launch_rmsnorm<T>(const float*, int, const float*, T*, int, int, int, float, \
                                    cudaStream_t);                                             \
    template void launch_merge_out<T>(const float*, int, const int32_t*, const float*, int,    \
                                      size_t, const float*, const float*, int, size_t, int,    \
                                      float, float*, const float*, T*, float, int, int, int,   \
                                      cudaStream_t);                                           \
    template void launch_state_merge<T>(const float*, const float*, int, size_t, float*,      \
                                        float*, int32_t*, int, const float*, int, const float*, \
                                        T*, int, int, float, cudaStream_t);                    \
    template void launch_merge_input<T>(const float*, int, const int32_t*, const float*,       \
                                        const float*, T*, int, int, int, float, cudaStream_t); \
    template void launch_qkv_dec<T>(const float*, int, size_t, const int32_t*, RopeTab, float*, \
                                    T*, T*, int, int, int, int, cudaStream_t);                 \
    template void launch_add_rmsnorm<T>(float*, const float*, int, size_t, const float*, T*,   \
                                        int, int, float, cudaStream_t);                        \
    template void launch_qkv_enc<T>(const float*, const int32_t*, RopeTab, float*, T*, size_t, \
                                    int, int, int, int, int, cudaStream_t);                    \
    template void launch_mem_scatter<T>(const float*, const int32_t*, RopeTab, T*, size_t, int,\
                                        int, int, int, int, cudaStream_t);                     \
    template void launch_swiglu<T>(const float*, int, size_t, int, T*, int, cudaStream_t);     \
    template void launch_ring_write<T>(const T*, const T*, const int32_t*, T*, size_t, int,    \
                                       int, int, int, int, cudaStream_t);
RLT_INST(float)
RLT_INST(bf16)
#undef RLT_INST

}  // namespace rlt
