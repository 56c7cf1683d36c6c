// Launchers of the RLT kernels (host side).  Every launcher enqueues on
// `st` and counts its launches; none synchronises.
//
// Row conventions: a call that handles n positions per sequence for B
// sequences works on R = B*n "rows" r = b*n + i, position i of sequence b.
// pos[] arrays are the device copies of the per-sequence counters before the
// call (positions are 1-based: the i-th new position of sequence b is
// pos[b] + 1 + i).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace rlt {

// GEMM epilogues: C (fp32) = acc | C += acc | Ct (storage type) = acc |
// SwiGLU of interleaved W1;W3 columns | RoPE and cache scatter (RopeScatter)
enum GemmMode { kStoreF32 = 0, kAddF32 = 1, kStoreT = 2, kSwiGLU = 3, kRopeScatter = 4 };
// The fused FFN input projection stores W1 and W3 interleaved in blocks of
// kW13Block rows: packed rows [64k, 64k+32) are W1 rows [32k, 32k+32)
// (gates), rows [64k+32, 64k+64) the W3 rows of the same units, so any
// 64-column output tile holds 32 gates and their 32 up projections.
constexpr int kW13Block = 32;
__host__ __device__ __forceinline__ int w13_gate_col(int j) {
    return (j / kW13Block) * 2 * kW13Block + j % kW13Block;
}

struct RopeTab {          // cos/sin of p * base^(-2i/dh), p = 0..max_pos, i < dh/2
    const float* cs;      // [max_pos+1][dh/2] cos
    const float* sn;      // [max_pos+1][dh/2] sin
    int half;
    int max_pos;          // last position with a row in the tables
};

// Rotate-half RoPE of one pair (j, j + d_h/2) by the angle whose cosine and
// sine are c and s.  Written with explicit fused multiply-adds so that every
// kernel that rotates (the scatters, the attention kernels that form q and k
// themselves, the GEMM epilogue below) rounds alike.
__device__ __forceinline__ void rope_pair(float x1, float x2, float c, float s, float& y1,
                                          float& y2) {
    y1 = fmaf(x1, c, -(x2 * s));
    y2 = fmaf(x2, c, x1 * s);
}

// SwiGLU of one unit: SiLU(a) * u, a the gate pre-activation and u the up
// projection, with the fast exponential and division (a few ulp in fp32; the
// result is stored in bf16, or carries the fp32 models' 1e-4 tolerance).
// Every kernel that applies SwiGLU uses this one form.
__device__ __forceinline__ float silu_mul(float a, float u) {
    return __fdividef(a, 1.0f + __expf(-a)) * u;
}

// Destination of an encoder product whose GEMM epilogue applies RoPE and
// scatters the result (kRopeScatter): the columns are the q|k|v blocks
// (sec0 = 0) or the memory's k|v blocks (sec0 = 1), d columns each.  Row
// r = b*n + i is position pos[b] + 1 + i of sequence b: q goes rotated to
// Q[r][d] (fp32), k rotated and v as they are to the cache of row b
// (cache + b*row_stride: K [heads][T_cap][dh], then V), in bf16.
struct RopeScatter {
    float* Q;
    bf16* cache;
    size_t row_stride;
    int T_cap;
    const int32_t* pos;
    RopeTab rope;
    int n, dh, d, sec0;
};
// C = A . W^T with the kRopeScatter epilogue on the persistent tensor-core
// GEMM; false (nothing launched) where it does not apply (fewer than 2048
// rows, d not a multiple of 256, d_h not 64 or 128).
bool launch_gemm_rope_scatter(const bf16* A, int lda, const bf16* W, int ldw, int M, int N,
                              int K, const RopeScatter& rs, cudaStream_t st);

template <typename T>
void launch_embed(const T* E, const int32_t* tok, float* X, int R, int d, int vocab, int* err,
                  cudaStream_t st);
template <typename T>
void launch_rmsnorm(const float* X, int ldx, const float* gain, T* Y, int ldy, int R, int d,
                    float eps, cudaStream_t st);
// dispatcher: tensor-core kernel where it applies, CUDA-core kernel otherwise
template <typename T>
void launch_gemm(const T* A, int lda, const T* W, int ldw, float* C, int ldc, T* Ct, int ldct,
                 int M, int N, int K, int mode, cudaStream_t st);
// 2-D bf16 TMA map over a row-major [rows][cols] matrix of row pitch ld:
// boxes of 64 columns (128 bytes, swizzled) x box_rows rows (k_gemm_tc.cu).
bool make_tma_2d_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld,
                      int box_rows);
// Hd[M, N/2] = SwiGLU of A . W13^T (interleaved W13, N = 2 f_pad) in the
// tensor-core GEMM's epilogue; false (nothing launched) where unsupported.
bool launch_gemm_swiglu(const bf16* A, int lda, const bf16* W13, int ldw, bf16* Hd, int ldh, int M,
                        int N, int K, cudaStream_t st);
template <typename T>
int launch_gemm_split(const T* A, int lda, const T* W, int ldw, float* C, int ldc, int M, int N,
                      int K, int splits, size_t slab, cudaStream_t st);
template <typename T>
void launch_gemm_simt(const T* A, int lda, const T* W, int ldw, float* C, int ldc, T* Ct,
                      int ldct, int M, int N, int K, int mode, cudaStream_t st);

// merge: Gin[r] = [T(e_t), T(RMSNorm_s(fb[b]))], t = pos_dec[b]+1+i
template <typename T>
void launch_merge_input(const float* e, int T_cap, const int32_t* pos_dec, const float* fb,
                        const float* gain, T* Gin, int B, int n, int d, float eps, cudaStream_t st);
// z[r] = e_t + alpha * sigmoid(G[r] + bg) * S[r]   (S = W_s r); alpha ignored if G == nullptr.
// G and S may be split-K partial slabs (nG / nS slabs, slabG / slabS apart),
// rows ldg floats apart.  With a gain (non-null), also Y[r] = RMSNorm(z[r]) * gain.
template <typename T>
void launch_merge_out(const float* e, int T_cap, const int32_t* pos_dec, const float* G, int nG,
                      size_t slabG, const float* bg, const float* S, int nS, size_t slabS,
                      int ldg, float alpha, float* z, const float* gain, T* Y, float eps, int B,
                      int n, int d, cudaStream_t st);
// z += sum of residual partial slabs P (P may be null), then Y = RMSNorm(z)
template <typename T>
void launch_add_rmsnorm(float* Z, const float* P, int S, size_t slab, const float* gain, T* Y,
                        int R, int d, float eps, cudaStream_t st);

// decoder q/k/v: QKV fp32 [R][3d] -> Q fp32 [R][d] (RoPE), Kc, Vc storage [R][d] (RoPE on k)
template <typename T>
void launch_qkv_dec(const float* QKV, int S, size_t slab, const int32_t* pos_dec, RopeTab rope,
                    float* Q, T* Kc, T* Vc, int B, int n, int heads, int dh, cudaStream_t st);
// encoder q/k/v: q -> Q (RoPE); k (RoPE), v -> cache [b][2][h][T_cap][dh] + layer offset
template <typename T>
void launch_qkv_enc(const float* QKV, const int32_t* pos_enc, RopeTab rope, float* Q, T* cache,
                    size_t row_stride, int T_cap, int B, int n, int heads, int dh,
                    cudaStream_t st);
// memory: KV fp32 [R][2d] -> memory group g: [b][.. g ..][2][h][T_cap][dh] (RoPE on k)
template <typename T>
void launch_mem_scatter(const float* KV, const int32_t* pos_enc, RopeTab rope, T* mem,
                        size_t row_stride, int T_cap, int B, int n, int heads, int dh,
                        cudaStream_t st);
// Q fp32 [R][d] = RoPE(sum of the partial slabs P) at decoder positions
void launch_rope_q(const float* P, int S, size_t slab, float* Q, const int32_t* pos_dec,
                   RopeTab rope, int B, int n, int heads, int dh, cudaStream_t st);

template <typename T>
void launch_swiglu(const float* H, int S, size_t slab, int fpad, T* Hd, int R, cudaStream_t st);
void launch_copy_e(const float* X, const int32_t* pos_enc, float* e, int T_cap, int B, int n,
                   int d, cudaStream_t st);
// s[b] = z[b*n + n-1] (+ its residual partial slabs); RLT-2: R[b] = s[b] when
// (pos_dec[b]+n) % chunk == 0; with bump, then pos_dec[b] += n
void launch_set_state(const float* z, const float* P, int S, size_t slab, float* s, float* Rreg,
                      int32_t* pos_dec, int chunk, int B, int n, int d, bool bump,
                      cudaStream_t st);
void launch_pos_add(int32_t* pos, int B, int n, cudaStream_t st);
// one position per row: launch_set_state(bump) and the next launch_merge_input
template <typename T>
void launch_state_merge(const float* z, const float* P, int S, size_t slab, float* s, float* Rreg,
                        int32_t* pos_dec, int chunk, const float* e, int T_cap, const float* gain,
                        T* Gin, int B, int d, float eps, cudaStream_t st);
void launch_reset_rows(const int32_t* rows, int nrows, const float* s_star, float* s, float* Rr,
                       int32_t* pos_enc, int32_t* pos_dec, int d, cudaStream_t st);
template <typename T>
void launch_ring_write(const T* Kc, const T* Vc, const int32_t* pos_dec, T* ring,
                       size_t row_stride, int W, int B, int n, int heads, int dh,
                       cudaStream_t st);

// attention (one warp per row and head); outputs A storage [R][d]
template <typename T>
void launch_attn_enc(const float* Q, const T* cache, size_t row_stride, int T_cap,
                     const int32_t* pos_enc, T* A, int B, int n, int heads, int dh,
                     cudaStream_t st);
template <typename T>
void launch_attn_swa(const float* Q, const T* Kc, const T* Vc, const T* ring, size_t row_stride,
                     int W, const int32_t* pos_dec, T* A, int B, int n, int heads, int dh,
                     cudaStream_t st);
template <typename T>
void launch_attn_cross(const float* Q, const T* mem, size_t row_stride, int T_cap,
                       const int32_t* pos_dec, T* A, int B, int n, int heads, int dh,
                       cudaStream_t st);

// readout sampler: one block per row over logits fp32 [B][V]
void launch_sample(const float* logits, int V, int B, int32_t* argmax, int32_t* sampled,
                   uint64_t seed, uint64_t step, float temperature, cudaStream_t st);
// log softmax(logits/temperature) at ids[b * ids_stride] -> out[b * out_stride]
void launch_logprob(const float* logits, int V, int B, const int32_t* ids, int ids_stride,
                    float* out, int out_stride, float temperature, int* err, cudaStream_t st);

int read_and_clear_device_error();  // device error word of the bounded-wait kernels
int read_and_clear_attn_error();
int read_and_clear_persist_error();  // same, for the persistent GEMM
int read_and_clear_mq_error();       // same, for the multi-query block attention
int read_and_clear_sq_error();       // same, for the one-position attention
// Partial-sum slabs of a projection, consumed directly by an attention kernel.
struct ProjIn {
    const float* P;   // slab 0 of the fp32 partial sums, [R][ldp]
    int S;            // number of slabs, summed in slab order
    size_t slab;      // elements from one slab to the next
    int ldp;          // row pitch: 3d for the fused q|k|v projection, d for q alone
    RopeTab rope;
};
// bf16 decoder attention that forms q (and, for the window attention, the
// block's own k and v, which it then writes into the ring) from the
// projection slabs.  They return false, launching nothing, for shapes they do
// not handle; the caller then runs the RoPE scatter and the plain kernels.
bool launch_attn_swa_proj(const ProjIn& pin, bf16* ring, size_t row_stride, int W,
                          const int32_t* pos_dec, bf16* A, int B, int n, int heads, int dh,
                          cudaStream_t st);
bool launch_attn_cross_proj(const ProjIn& pin, const bf16* mem, size_t row_stride, int T_cap,
                            const int32_t* pos_dec, bf16* A, int B, int n, int heads, int dh,
                            cudaStream_t st);
bool fast_attn_enabled();           // false when RLT_ATTN=warp
// Blocks of 2..16 positions per row at d_h = 64 (k_attn_mq.cu): one warp per
// (row, head) scores the block's queries against 16-key tiles with the
// warp-level tensor-core MMA; the window form (SWA) also takes the block's
// own keys from the slabs and writes them into the ring.  false (nothing
// launched) for other shapes or when RLT_MQ=0.
// One position per row at d_h = 64 (k_attn_sq.cu): one warp per (row, head)
// streams 16-key tiles through shared memory by bulk copy and scores them on
// the CUDA cores (q and p fp32); false when RLT_SQ=0 or for other shapes.
template <bool SWA>
bool launch_attn_sq(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W,
                    bf16* A, int B, int heads, int dh, const ProjIn& pin, cudaStream_t st);
template <bool SWA>
bool launch_attn_mq(const bf16* base, size_t row_stride, int span, const int32_t* pos, int W,
                    bf16* A, int B, int n, int heads, int dh, const ProjIn& pin, cudaStream_t st);
// Encoder causal attention on the tensor cores: k_attn_enc_tc.cu (exact
// two-pass softmax) for d_h = 64 and at most 256 keys per row (max_keys =
// max over rows of pos_enc + n), k_attn_enc_fa.cu for longer prefixes and
// d_h = 128; false (nothing launched) for other head sizes.  err: the
// state's device error word.
bool launch_attn_enc_tc(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
                        const int32_t* pos, bf16* A, int B, int n, int heads, int dh, int max_keys,
                        int* err, cudaStream_t st);
// The same over prefixes of any length for d_h = 64 or 128 (k_attn_enc_fa.cu:
// key tiles of 128, running softmax, O accumulated in tensor memory); false
// (nothing launched) for other head sizes.
bool launch_attn_enc_fa(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
                        const int32_t* pos, bf16* A, int B, int n, int heads, int dh, int* err,
                        cudaStream_t st);
// The encoder's attention for one new position per row at d_h = 128 (the
// large model's generation steps): keys split over 4 warps per (row, head),
// q read rotated from Q; false (nothing launched) for other head sizes.
bool launch_attn_enc_step(const float* Q, const bf16* cache, size_t row_stride, int T_cap,
                          const int32_t* pos_enc, bf16* A, int B, int heads, int dh,
                          cudaStream_t st);
    // same, for the streaming attention kernels

// Failure-detection self-test (k_selftest.cu): one CTA whose single wait is
// never satisfied (kind 0: an mbarrier nobody arrives on; kind 1: a global
// word nobody sets), bounded by `polls` polls; on giving up it writes
// kDevTimeout to *err.
void launch_selftest_wait(int kind, uint32_t polls, int* err, cudaStream_t st);

// Debug builds (RLT_DEBUG=1): validate the rows' position counters before a
// transition block (encoding = false) or an encoder block of n positions
// (k_debug.cu); a no-op in other builds.
void launch_check_positions(const int32_t* pos_enc, const int32_t* pos_dec, int B, int n,
                            int T_cap, bool encoding, int* err, cudaStream_t st);

}  // namespace rlt
