// Shapes, shared-memory plan and launch parameters of the fused transition
// kernel (k_dec_fused.cu).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace rlt {
namespace fz {

constexpr int D = 512;        // model width
constexpr int H = 8;          // heads (= CTAs per cluster)
constexpr int DH = 64;        // head size
constexpr int FP = 1408;      // FFN width padded to 64
constexpr int NCH_F = FP / 64;
constexpr int RB = 16;        // sequences per cluster (MMA N)
constexpr int CL = 8;         // cluster size
constexpr int NT = 320;       // warp 0 TMA, warp 1 MMA, warps 2-9 compute
constexpr int NSLOT = 10;     // weight-box ring
constexpr int SLOT = 8192;    // one 64 x 64 bf16 box

constexpr int CHUNK_BYTES = RB * 128;              // one K-chunk of the B operand
constexpr int LAND_BYTES = CL * RB * 64 * 4;       // one landing zone (fp32 [8][16][64])
constexpr int OFF_STAGE = 0;
constexpr int OFF_OPND = NSLOT * SLOT;             // B operand, 16 chunks (K <= 1024)
constexpr int OFF_HID = OFF_OPND + 16 * CHUNK_BYTES;  // W_2 operand: this CTA's hidden chunks
constexpr int OFF_LAND = OFF_HID + 3 * CHUNK_BYTES;   // two landing zones
constexpr int OFF_Z = OFF_LAND + 2 * LAND_BYTES;   // residual slice fp32 [16][64]
constexpr int OFF_E = OFF_Z + RB * 64 * 4;         // e_t slice
constexpr int OFF_Q = OFF_E + RB * 64 * 4;         // q, k, v of head c
constexpr int OFF_K = OFF_Q + RB * 64 * 4;
constexpr int OFF_V = OFF_K + RB * 64 * 4;
constexpr int SMEM_USED = OFF_V + RB * 64 * 4;
constexpr int SMEM_DYN = SMEM_USED + 1024;         // + alignment slack
constexpr int TMEM_COLS = 128;
static_assert(OFF_OPND % 1024 == 0 && OFF_HID % 1024 == 0 && OFF_LAND % 1024 == 0, "alignment");
static_assert(SMEM_DYN <= 227 * 1024, "shared memory");

struct FusedParams {
    // weight maps (bf16, 64 x 64 boxes, 128-byte swizzle); decoder kinds span all layers
    CUtensorMap m_qkv;   // [L*3*512][512]
    CUtensorMap m_o;     // [L*512][512]
    CUtensorMap m_xq;    // [L*512][512]
    CUtensorMap m_xo;    // [L*512][512]
    CUtensorMap m_13;    // [L*2*1408][512]  (W1 rows, then W3 rows, per layer)
    CUtensorMap m_2;     // [L*512][1408]
    CUtensorMap m_g;     // [512][1024]  merge gate W_g
    CUtensorMap m_s;     // [512][512]   merge projection W_s
    const float* e;      // [B][T_cap][512]
    float* s;            // [B][512]
    int32_t* pos_dec;    // [B]
    int* err;            // sticky error word
    const bf16* mem;     // [B][G][2][8][T_cap][64]
    bf16* ring;          // [B][L][2][8][W-1][64]
    const float* rope_cs;  // [T_cap+1][32]
    const float* rope_sn;
    const float* g_swa;  // [L][512]
    const float* g_x;
    const float* g_ffn;
    const float* g_merge;  // [512]
    const float* bg;       // [512]
    size_t mem_row, ring_row;   // elements per sequence
    int B, T_cap, L, W, G, nsteps, variant;
    float alpha, eps;
};

}  // namespace fz

bool launch_dec_fused(const fz::FusedParams& p, cudaStream_t st);
bool make_tma_2d_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld,
                      int box_rows);

}  // namespace rlt
