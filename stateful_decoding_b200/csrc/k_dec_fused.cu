// The RLT-1 transition, fused: merge gate, L_D decoder blocks (window
// self-attention with in-place ring update, cross-attention to M_{<=t},
// SwiGLU FFN, residuals and RMSNorms) and the state hand-off, for nsteps
// consecutive positions, in one launch (greeksharifa "Recurrent Looped
// Transformer 요약 설명" §2.3-§2.5; jiphyeonjeon review "Recurrent Looped
// Transformer" §3.1-§3.3 and §5: transitions of independent sequences batch
// together, each sequence keeping its own caches).
//
// Shape handled: bf16 storage, d = 512, 8 heads of 64, FFN padded to 1408,
// window W <= 65, memory groups 1 or L_D.
//
// Organisation.  A cluster of 8 CTAs owns 16 sequences ("rows") and runs all
// steps for them; clusters never wait for one another.  CTA c owns head c and
// the feature slice [64c, 64c+64) of every d-wide vector: it keeps that slice
// of the residual stream z in shared memory, computes those output features
// of every projection (the weight rows of the slice), and runs the window
// and cross attention of head c.  Full-row inputs (RMSNorm over all 512
// features, attention outputs of all heads) are exchanged through distributed
// shared memory: each CTA writes its slice into every peer's landing zone,
// then the cluster synchronises.  W_2 is split along its input (hidden)
// dimension instead: each CTA forms partial sums for all 512 outputs from its
// own hidden units and the partials are reduced at their owners in a fixed
// order.
//
// Warp roles: warp 0 streams weight boxes (64 rows x 64 columns, bf16) with
// TMA into a 10-slot ring, running ahead of the arithmetic through the whole
// fixed schedule; warp 1 issues the tensor-core MMAs (one thread): each
// 64-row weight box is the A operand of an M=128 tcgen05 MMA (rows 64-127 of
// the tile are not used), the 16 rows' activations (bf16, K-major, 128-byte
// swizzle) the B operand (N = 16); fp32 accumulators live in TMEM.  Warps
// 2-9 do everything else.  All waits are bounded; a wait that gives up sets
// the state's error word and lets the CTA run to its end.
#include <cuda.h>
#include <math.h>

#include "fused.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace rlt {
namespace fz {

using namespace tc;

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void remote_arrive(uint32_t cl_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr)
                 : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void cluster_barrier_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
__device__ __forceinline__ void fence_cluster() {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bar_compute() {   // the 8 compute warps only
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

__device__ __forceinline__ float bf16r(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
// byte offset of 16-byte unit u of row r inside a 128-byte-swizzled K-chunk tile
__device__ __forceinline__ uint32_t swz(int r, int u) {
    return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
}

// ---------------------------------------------------------------- schedule
enum JobKind { J_MERGE = 0, J_QKV = 1, J_WO = 2, J_XQ = 3, J_XO = 4, J_W13 = 5, J_W2 = 6 };

__device__ __forceinline__ int nhid(int c) { return c < (NCH_F - 2 * CL) ? 3 : 2; }

__device__ __forceinline__ int ntiles(int kind, int c) {
    switch (kind) {
        case J_MERGE: return 2;
        case J_QKV: return 3;
        case J_W13: return 2 * nhid(c);
        case J_W2: return 8;
        default: return 1;
    }
}

struct TileRef {
    const CUtensorMap* map;
    int row;      // first weight row of the 64-row box
    int nch;      // K-chunks
    int kx0;      // K coordinate (elements) of chunk 0
    int kstep;    // K coordinate step per chunk
    int op0;      // first operand chunk
    bool hid;     // operand from the hidden buffer
};

__device__ __forceinline__ TileRef tile_of(const FusedParams& P, int kind, int l, int t, int c) {
    TileRef r;
    r.kx0 = 0;
    r.kstep = 64;
    r.op0 = 0;
    r.hid = false;
    r.nch = D / 64;
    switch (kind) {
        case J_MERGE:
            if (t == 0) { r.map = &P.m_g; r.row = c * 64; r.nch = 2 * D / 64; }
            else { r.map = &P.m_s; r.row = c * 64; r.op0 = D / 64; }
            break;
        case J_QKV: r.map = &P.m_qkv; r.row = l * 3 * D + t * D + c * 64; break;
        case J_WO: r.map = &P.m_o; r.row = l * D + c * 64; break;
        case J_XQ: r.map = &P.m_xq; r.row = l * D + c * 64; break;
        case J_XO: r.map = &P.m_xo; r.row = l * D + c * 64; break;
        case J_W13: {
            const int i = t >> 1, which = t & 1, j = c + CL * i;
            r.map = &P.m_13;
            r.row = l * 2 * FP + j * 128 + which * 64;     // interleaved W1;W3 blocks
            break;
        }
        default: {  // J_W2: output rows t*64.., K over this CTA's hidden chunks c, c+8, c+16
            r.map = &P.m_2;
            r.row = l * D + t * 64;
            r.nch = nhid(c);
            r.kx0 = c * 64;
            r.kstep = CL * 64;
            r.hid = true;
            break;
        }
    }
    return r;
}

// One accumulator per tile.  (Measured on B200: spreading a tile's K range
// over several partial accumulators, or interleaving tiles chunk by chunk,
// made the MMA issue slower, not faster; so did releasing weight slots in
// batches.  A 64-wide K chunk costs ~0.4 us of issue time at N = 16.)
__device__ __forceinline__ int nsplit(int) { return 1; }
__device__ __forceinline__ int kfirst(int kind, int t) { return (kind == J_MERGE && t == 1) ? 8 : 0; }
__device__ __forceinline__ int nch_max(int kind, int c) {
    return kind == J_MERGE ? 2 * D / 64 : (kind == J_W2 ? nhid(c) : D / 64);
}

__device__ __forceinline__ int njobs(const FusedParams& P) { return 1 + 6 * P.L; }
__device__ __forceinline__ void job_kind(int j, int& kind, int& l) {
    if (j == 0) { kind = J_MERGE; l = 0; }
    else { kind = 1 + (j - 1) % 6; l = (j - 1) / 6; }
}

// ---------------------------------------------------------------- shared state
struct Ctl {
    uint64_t full[NSLOT], empty[NSLOT];
    uint64_t op_full, acc_full;
    uint64_t clbar[2];
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool waitb(uint64_t* bar, uint32_t parity, Ctl* ctl, int* err) {
    if (ctl->abort) return false;
    for (uint32_t i = 0; i < (1u << 24); ++i)
        if (mbar_try(bar, parity)) return true;
    ctl->abort = 1;
    atomicExch(err, kDevTimeout);
    return false;
}

// Cluster-wide sync of the compute warps (double-buffered remote mbarriers:
// a CTA can only arrive for phase k+2 after every CTA arrived for phase k+1).
__device__ __forceinline__ void cl_sync(Ctl* ctl, uint32_t& cph, int ct, int* err) {
    bar_compute();
    uint64_t* bar = &ctl->clbar[cph & 1];
    if (ct == 0) {
        fence_cluster();
        const uint32_t a = smem_u32(bar);
        for (uint32_t dst = 0; dst < CL; ++dst) remote_arrive(mapa(a, dst));
    }
    const uint32_t par = (cph >> 1) & 1u;
    if (!ctl->abort) {
        bool ok = false;
        for (uint32_t i = 0; i < (1u << 24) && !ok; ++i) ok = try_wait_cluster(bar, par);
        if (!ok) {
            ctl->abort = 1;
            atomicExch(err, kDevTimeout);
        }
    }
    ++cph;
}

// ---------------------------------------------------------------- compute helpers
// Send my 64-feature fp32 slice of 16 rows to every CTA's landing zone:
// land[src = me][r][0..63].  Thread (r, q) sends features 4q..4q+3.
__device__ __forceinline__ void bcast_slice_f32(const float* zs, uint8_t* land, int c, int r,
                                                int q) {
    const float4 v = *reinterpret_cast<const float4*>(zs + r * 64 + q * 4);
    const uint32_t a = smem_u32(land + ((c * RB + r) * 64 + q * 4) * 4);
    const uint4 u = make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                               __float_as_uint(v.w));
#pragma unroll
    for (uint32_t dst = 0; dst < CL; ++dst) st_cluster_v4(mapa(a, dst), u);
}

// Full-row RMSNorm of land (fp32 [8][16][64] = rows of 512) into the operand
// buffer, chunks op0 .. op0+7: thread (r, q) owns features 32q..32q+31.
__device__ __forceinline__ void norm_to_operand(const uint8_t* land, const float* gain, float eps,
                                                uint8_t* opnd, int op0, int r, int q) {
    const float* x = reinterpret_cast<const float*>(land) + ((q >> 1) * RB + r) * 64 + (q & 1) * 32;
    float v[32];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const float4 t = *reinterpret_cast<const float4*>(x + i);
        v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) ss += v[i] * v[i];
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss / (float)D + eps);
    const float* g = gain + q * 32;
    uint8_t* chunk = opnd + (op0 + (q >> 1)) * CHUNK_BYTES;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * u + 0] * inv * g[8 * u + 0], v[8 * u + 1] * inv * g[8 * u + 1]);
        w.y = pack_bf16x2(v[8 * u + 2] * inv * g[8 * u + 2], v[8 * u + 3] * inv * g[8 * u + 3]);
        w.z = pack_bf16x2(v[8 * u + 4] * inv * g[8 * u + 4], v[8 * u + 5] * inv * g[8 * u + 5]);
        w.w = pack_bf16x2(v[8 * u + 6] * inv * g[8 * u + 6], v[8 * u + 7] * inv * g[8 * u + 7]);
        *reinterpret_cast<uint4*>(chunk + swz(r, (q & 1) * 4 + u)) = w;
    }
}

// Copy the bf16 landing zone ([8 heads][16][64]) into operand chunks 0..7.
__device__ __forceinline__ void bf16_land_to_operand(const uint8_t* land, uint8_t* opnd, int r,
                                                     int q) {
    const uint8_t* src = land + (((q >> 1) * RB + r) * 64 + (q & 1) * 32) * 2;
    uint8_t* chunk = opnd + (q >> 1) * CHUNK_BYTES;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(chunk + swz(r, (q & 1) * 4 + u)) =
            *reinterpret_cast<const uint4*>(src + u * 16);
}

// One attention row on a warp: LPK = 8 lanes per key (16 bytes each), 4 keys
// per warp-wide load, blocks of 32 keys; online softmax; optionally one extra
// key (the current position) from shared memory.  Output: o[64] (fp32) in
// lanes 0..7 (8 values each) after the group reduction.
template <bool RING>
__device__ __forceinline__ void attend_row(const float* q_s, const bf16* kb, const bf16* vb,
                                           int nkeys, int p_first, int ring_slots,
                                           const float* kcur, const float* vcur, float (&out)[8],
                                           int lane) {
    const int seg = lane & 7, grp = lane >> 3;
    float q[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) q[x] = q_s[seg * 8 + x];
    float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) acc[x] = 0.f;
    for (int j0 = 0; j0 < nkeys; j0 += 32) {
        uint4 kr[8], vr[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int idx = j0 + j * 4 + grp;
            if (idx < nkeys) {
                const int p = p_first + idx;                       // 1-based position
                const size_t off = RING ? (size_t)((p - 1) % ring_slots) * 64 : (size_t)(p - 1) * 64;
                kr[j] = *reinterpret_cast<const uint4*>(kb + off + seg * 8);
                vr[j] = *reinterpret_cast<const uint4*>(vb + off + seg * 8);
            } else {
                kr[j] = make_uint4(0, 0, 0, 0);
                vr[j] = make_uint4(0, 0, 0, 0);
            }
        }
        float s[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float kf[8];
            unpack8(kr[j], kf);
            float dot = 0.f;
#pragma unroll
            for (int x = 0; x < 8; ++x) dot = fmaf(q[x], kf[x], dot);
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            dot += __shfl_xor_sync(0xffffffffu, dot, 4);
            s[j] = (j0 + j * 4 + grp < nkeys) ? dot : -INFINITY;
        }
        float bm = s[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) bm = fmaxf(bm, s[j]);
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
        const float mn = fmaxf(m, bm);
        const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
        float ps = 0.f, pj[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            pj[j] = (s[j] == -INFINITY) ? 0.f : expf(s[j] - mn);
            ps += pj[j];
        }
        ps += __shfl_xor_sync(0xffffffffu, ps, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
        l = l * corr + ps;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] *= corr;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float vf[8];
            unpack8(vr[j], vf);
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = fmaf(pj[j], vf[x], acc[x]);
        }
        m = mn;
    }
    if (kcur) {   // the current position's key/value (window attention)
        float dot = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) dot = fmaf(q[x], kcur[seg * 8 + x], dot);
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        dot += __shfl_xor_sync(0xffffffffu, dot, 4);
        const float mn = fmaxf(m, dot);
        const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
        const float p = expf(dot - mn);
        l = l * corr + p;
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] = acc[x] * corr + (grp == 0 ? p * vcur[seg * 8 + x] : 0.f);
        m = mn;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x) {
        acc[x] += __shfl_xor_sync(0xffffffffu, acc[x], 8);
        acc[x] += __shfl_xor_sync(0xffffffffu, acc[x], 16);
    }
    const float inv = 1.0f / l;
#pragma unroll
    for (int x = 0; x < 8; ++x) out[x] = acc[x] * inv;
}

// Tile t's accumulator for this warp's lane quarter: the sum, in order, of
// its ns partial accumulators (TMEM columns (t*ns + s) * 16).
__device__ __forceinline__ void acc_sum(uint32_t tmem, int quarter, int t, int ns,
                                        float (&v)[16]) {
    const uint32_t base = tmem + ((uint32_t)(32 * quarter) << 16);
    tmem_ld16(base + (uint32_t)(t * ns * RB), v);
    for (int s = 1; s < ns; ++s) {
        float w[16];
        tmem_ld16(base + (uint32_t)((t * ns + s) * RB), w);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] += w[i];
    }
}

// ---------------------------------------------------------------- the kernel
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(NT, 1)
k_dec_fused(const __grid_constant__ FusedParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ Ctl ctl;
    __shared__ int pos_s[RB];     // positions (pos_dec) of the cluster's rows at launch
    uint8_t* stage = sm + OFF_STAGE;
    uint8_t* opnd = sm + OFF_OPND;
    uint8_t* hidb = sm + OFF_HID;
    uint8_t* land0 = sm + OFF_LAND;
    float* zs = reinterpret_cast<float*>(sm + OFF_Z);
    float* es = reinterpret_cast<float*>(sm + OFF_E);
    float* qs = reinterpret_cast<float*>(sm + OFF_Q);
    float* ks = reinterpret_cast<float*>(sm + OFF_K);
    float* vs = reinterpret_cast<float*>(sm + OFF_V);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = (int)cluster_rank();
    const int row0 = (int)cluster_id_x() * RB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
        }
        mbar_init(&ctl.op_full, 1);
        mbar_init(&ctl.acc_full, 1);
        mbar_init(&ctl.clbar[0], CL);
        mbar_init(&ctl.clbar[1], CL);
        ctl.abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < RB) {
        const int bb = (int)cluster_id_x() * RB + threadIdx.x;
        pos_s[threadIdx.x] = bb < P.B ? P.pos_dec[bb] : 0;
    }
    if (warp == 1) tmem_alloc(&ctl.tmem_base, TMEM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    cluster_barrier_all();        // peers' barriers are initialised before any remote arrive
    const uint32_t tmem = ctl.tmem_base;
    const int NJ = njobs(P);
    const int j_begin = P.variant == 0 ? 1 : 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_map(&P.m_qkv); prefetch_map(&P.m_o); prefetch_map(&P.m_xq);
            prefetch_map(&P.m_xo); prefetch_map(&P.m_13); prefetch_map(&P.m_2);
            prefetch_map(&P.m_g); prefetch_map(&P.m_s);
            uint32_t ld = 0;
            for (int step = 0; step < P.nsteps && !ctl.abort; ++step)
                for (int j = j_begin; j < NJ && !ctl.abort; ++j) {
                    int kind, l;
                    job_kind(j, kind, l);
                    const int nt = ntiles(kind, c);
                    for (int t = 0; t < nt && !ctl.abort; ++t)
                        for (int kl = 0; kl < tile_of(P, kind, l, t, c).nch && !ctl.abort; ++kl) {
                            const TileRef tr = tile_of(P, kind, l, t, c);
                            const int s = ld % NSLOT;
                            const uint32_t ph = (ld / NSLOT) & 1u;
                            if (ld >= NSLOT && !waitb(&ctl.empty[s], ph ^ 1u, &ctl, P.err)) break;
                            mbar_expect_tx(&ctl.full[s], SLOT);
                            tma_load_2d(stage + s * SLOT, tr.map, tr.kx0 + kl * tr.kstep, tr.row,
                                        &ctl.full[s]);
                            ++ld;
                        }
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, RB);
            uint32_t ld = 0, job = 0;
            for (int step = 0; step < P.nsteps; ++step)
                for (int j = j_begin; j < NJ; ++j, ++job) {
                    int kind, l;
                    job_kind(j, kind, l);
                    if (!waitb(&ctl.op_full, job & 1u, &ctl, P.err)) continue;
                    fence_after_sync();
                    const int nt = ntiles(kind, c), nk = nch_max(kind, c), ns = nsplit(kind);
                    (void)nk;
                    // slot releases are batched: a commit per consumed box costs a
                    // pipe round trip, so up to kBatch boxes are released together
                    constexpr int kBatch = 1;
                    int pend[kBatch], np = 0;
                    for (int t = 0; t < nt; ++t) {
                        const TileRef tr = tile_of(P, kind, l, t, c);
                        for (int kl = 0; kl < tr.nch; ++kl) {
                            const int s = ld % NSLOT;
                            const uint32_t ph = (ld / NSLOT) & 1u;
                            ++ld;
                            // TMA data is ordered by the barrier's transaction count:
                            // no tcgen05 fence is needed between the wait and the MMA
                            if (!waitb(&ctl.full[s], ph, &ctl, P.err)) continue;
                            const uint32_t a = smem_u32(stage + s * SLOT);
                            const uint32_t bsm =
                                smem_u32((tr.hid ? hidb : opnd) + (tr.op0 + kl) * CHUNK_BYTES);
                            const uint32_t col = (uint32_t)((t * ns + kl % ns) * RB);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_bf16(tmem + col, sdesc_k_sw128(a + kk * 32),
                                         sdesc_k_sw128(bsm + kk * 32), idesc,
                                         (kl < ns && kk == 0) ? 0u : 1u);
                            pend[np++] = s;
                            if (np == kBatch) {
                                for (int i = 0; i < kBatch; ++i) mma_commit(&ctl.empty[pend[i]]);
                                np = 0;
                            }
                        }
                    }
                    for (int i = 0; i < np; ++i) mma_commit(&ctl.empty[pend[i]]);
                    mma_commit(&ctl.acc_full);
                }
        }
    } else {
        // ------------------------------------------------ compute warps
        const int ct = threadIdx.x - 64;        // 0..255
        const int r = ct >> 4, q = ct & 15;     // row, quarter-of-slice (4 features)
        const int b = row0 + r;
        const bool valid = b < P.B;
        const int cw = warp - 2;                // 0..7
        const int quarter = warp & 3;           // TMEM lane quarter of this warp
        const bool epi_a = (warp == 4 || warp == 5), epi_b = (warp == 8 || warp == 9);
        const int f_epi = (quarter & 1) * 32 + lane;   // feature of the epilogue thread
        const int pos0 = pos_s[r];
        {
            float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            if (valid) z = *reinterpret_cast<const float4*>(P.s + (size_t)b * D + c * 64 + q * 4);
            *reinterpret_cast<float4*>(zs + r * 64 + q * 4) = z;
        }
        bar_compute();
        uint32_t job = 0, cph = 0;
        int par = 0;                            // landing zone in use
        const int W = P.W, slots = P.W - 1;

        auto land = [&](int p) { return land0 + p * LAND_BYTES; };
        auto signal_operand = [&]() {
            fence_proxy_async();
            bar_compute();
            if (ct == 0) mbar_arrive(&ctl.op_full);
        };
        auto wait_acc = [&]() {
            waitb(&ctl.acc_full, job & 1u, &ctl, P.err);
            fence_after_sync();
        };
        auto done_acc = [&]() {
            fence_before_sync();
            bar_compute();
            ++job;
        };

        for (int step = 0; step < P.nsteps; ++step) {
            // per-row position of this step (1-based); rows past B use t = 1
            const int t_of_r = valid ? pos0 + 1 + step : 1;
            // ----------------------------------------- merge (RLT-1)
            if (P.variant != 0) {
                bcast_slice_f32(zs, land(par), c, r, q);
                {   // e_t: full row into operand chunks 0..7 (bf16), my slice kept in fp32
                    const float* er = P.e + ((size_t)(valid ? b : 0) * P.T_cap + (t_of_r - 1)) * D + q * 32;
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 x4 = valid ? *reinterpret_cast<const float4*>(er + i)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                        v[i] = x4.x; v[i + 1] = x4.y; v[i + 2] = x4.z; v[i + 3] = x4.w;
                    }
                    uint8_t* chunk = opnd + (q >> 1) * CHUNK_BYTES;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 w;
                        w.x = pack_bf16x2(v[8 * u], v[8 * u + 1]);
                        w.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
                        w.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
                        w.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
                        *reinterpret_cast<uint4*>(chunk + swz(r, (q & 1) * 4 + u)) = w;
                    }
                    if ((q >> 1) == c) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) es[r * 64 + (q & 1) * 32 + i] = v[i];
                    }
                }
                cl_sync(&ctl, cph, ct, P.err);
                norm_to_operand(land(par), P.g_merge, P.eps, opnd, D / 64, r, q);
                par ^= 1;
                signal_operand();
                wait_acc();
                if (epi_a) {
                    float g[16], w[16];
                    acc_sum(tmem, quarter, 0, nsplit(J_MERGE), g);
                    acc_sum(tmem, quarter, 1, nsplit(J_MERGE), w);
                    const float bgf = P.bg[c * 64 + f_epi];
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) {
                        const float gate = 1.0f / (1.0f + expf(-(g[rr] + bgf)));
                        zs[rr * 64 + f_epi] = es[rr * 64 + f_epi] + P.alpha * gate * w[rr];
                    }
                }
                done_acc();
            } else {
                const float* er = P.e + ((size_t)(valid ? b : 0) * P.T_cap + (t_of_r - 1)) * D + c * 64 + q * 4;
                float4 x4 = valid ? *reinterpret_cast<const float4*>(er) : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(zs + r * 64 + q * 4) = x4;
                bar_compute();
            }

            for (int l = 0; l < P.L; ++l) {
                const int g = P.G > 1 ? l : 0;
                // ------------------------------------- window self-attention
                bcast_slice_f32(zs, land(par), c, r, q);
                cl_sync(&ctl, cph, ct, P.err);
                norm_to_operand(land(par), P.g_swa + l * D, P.eps, opnd, 0, r, q);
                par ^= 1;
                signal_operand();
                wait_acc();
                if (epi_a || epi_b) {
                    float v[16];
                    // pair a: tiles 0 (q) and 2 (v); pair b: tile 1 (k)
                    if (epi_a) {
                        acc_sum(tmem, quarter, 0, nsplit(J_QKV), v);
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) qs[rr * 64 + f_epi] = v[rr];
                        acc_sum(tmem, quarter, 2, nsplit(J_QKV), v);
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) vs[rr * 64 + f_epi] = bf16r(v[rr]);
                    } else {
                        acc_sum(tmem, quarter, 1, nsplit(J_QKV), v);
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) ks[rr * 64 + f_epi] = v[rr];
                    }
                }
                done_acc();
                {   // RoPE at t on q and k: thread (r, q) turns pairs 2q, 2q+1
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = q * 2 + jj;
                        const float cs = P.rope_cs[(size_t)t_of_r * 32 + j];
                        const float sn = P.rope_sn[(size_t)t_of_r * 32 + j];
                        float x1 = qs[r * 64 + j], x2 = qs[r * 64 + j + 32];
                        qs[r * 64 + j] = (x1 * cs - x2 * sn) * 0.125f;
                        qs[r * 64 + j + 32] = (x2 * cs + x1 * sn) * 0.125f;
                        x1 = ks[r * 64 + j];
                        x2 = ks[r * 64 + j + 32];
                        ks[r * 64 + j] = bf16r(x1 * cs - x2 * sn);
                        ks[r * 64 + j + 32] = bf16r(x2 * cs + x1 * sn);
                    }
                }
                bar_compute();
                // attention of head c for rows 2cw, 2cw+1
                for (int rr = 2 * cw; rr < 2 * cw + 2; ++rr) {
                    const int bb = row0 + rr;
                    const bool vr_ = bb < P.B;
                    const int tt = vr_ ? pos_s[rr] + 1 + step : 1;
                    float o[8];
                    const int nring = vr_ ? min(tt - 1, slots) : 0;
                    const bf16* kb = P.ring + (size_t)(vr_ ? bb : 0) * P.ring_row + ((size_t)(l * 2 + 0) * H + c) * (slots > 0 ? slots : 1) * 64;
                    const bf16* vb = P.ring + (size_t)(vr_ ? bb : 0) * P.ring_row + ((size_t)(l * 2 + 1) * H + c) * (slots > 0 ? slots : 1) * 64;
                    attend_row<true>(qs + rr * 64, kb, vb, nring, tt - nring, slots > 0 ? slots : 1,
                                     ks + rr * 64, vs + rr * 64, o, lane);
                    if (lane < 8) {
                        uint4 w;
                        w.x = pack_bf16x2(o[0], o[1]);
                        w.y = pack_bf16x2(o[2], o[3]);
                        w.z = pack_bf16x2(o[4], o[5]);
                        w.w = pack_bf16x2(o[6], o[7]);
                        const uint32_t a = smem_u32(land(par) + ((c * RB + rr) * 64 + lane * 8) * 2);
#pragma unroll
                        for (uint32_t dst = 0; dst < CL; ++dst) st_cluster_v4(mapa(a, dst), w);
                    }
                }
                bar_compute();
                // ring update: the current k, v into slot (t-1) mod (W-1), after every read
                if (W > 1 && valid) {
                    const int slot = (t_of_r - 1) % slots;
                    const int u = q & 7;
                    const float* src = (q < 8 ? ks : vs) + r * 64 + u * 8;
                    uint4 w;
                    w.x = pack_bf16x2(src[0], src[1]);
                    w.y = pack_bf16x2(src[2], src[3]);
                    w.z = pack_bf16x2(src[4], src[5]);
                    w.w = pack_bf16x2(src[6], src[7]);
                    bf16* dstp = P.ring + (size_t)b * P.ring_row +
                                 ((size_t)(l * 2 + (q < 8 ? 0 : 1)) * H + c) * slots * 64 +
                                 (size_t)slot * 64 + u * 8;
                    *reinterpret_cast<uint4*>(dstp) = w;
                }
                cl_sync(&ctl, cph, ct, P.err);
                bf16_land_to_operand(land(par), opnd, r, q);
                par ^= 1;
                signal_operand();
                wait_acc();
                if (epi_a) {
                    float v[16];
                    acc_sum(tmem, quarter, 0, nsplit(J_WO), v);
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) zs[rr * 64 + f_epi] += v[rr];
                }
                done_acc();
                // ------------------------------------- cross-attention
                bcast_slice_f32(zs, land(par), c, r, q);
                cl_sync(&ctl, cph, ct, P.err);
                norm_to_operand(land(par), P.g_x + l * D, P.eps, opnd, 0, r, q);
                par ^= 1;
                signal_operand();
                wait_acc();
                if (epi_a) {
                    float v[16];
                    acc_sum(tmem, quarter, 0, nsplit(J_WO), v);
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) qs[rr * 64 + f_epi] = v[rr];
                }
                done_acc();
                {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = q * 2 + jj;
                        const float cs = P.rope_cs[(size_t)t_of_r * 32 + j];
                        const float sn = P.rope_sn[(size_t)t_of_r * 32 + j];
                        const float x1 = qs[r * 64 + j], x2 = qs[r * 64 + j + 32];
                        qs[r * 64 + j] = (x1 * cs - x2 * sn) * 0.125f;
                        qs[r * 64 + j + 32] = (x2 * cs + x1 * sn) * 0.125f;
                    }
                }
                bar_compute();
                for (int rr = 2 * cw; rr < 2 * cw + 2; ++rr) {
                    const int bb = row0 + rr;
                    const bool vr_ = bb < P.B;
                    const int tt = vr_ ? pos_s[rr] + 1 + step : 0;
                    const bf16* kb = P.mem + (size_t)(vr_ ? bb : 0) * P.mem_row +
                                     ((size_t)(g * 2 + 0) * H + c) * P.T_cap * 64;
                    const bf16* vb = P.mem + (size_t)(vr_ ? bb : 0) * P.mem_row +
                                     ((size_t)(g * 2 + 1) * H + c) * P.T_cap * 64;
                    float o[8];
                    attend_row<false>(qs + rr * 64, kb, vb, tt, 1, 1, nullptr, nullptr, o, lane);
                    if (!vr_) {
#pragma unroll
                        for (int x = 0; x < 8; ++x) o[x] = 0.f;
                    }
                    if (lane < 8) {
                        uint4 w;
                        w.x = pack_bf16x2(o[0], o[1]);
                        w.y = pack_bf16x2(o[2], o[3]);
                        w.z = pack_bf16x2(o[4], o[5]);
                        w.w = pack_bf16x2(o[6], o[7]);
                        const uint32_t a = smem_u32(land(par) + ((c * RB + rr) * 64 + lane * 8) * 2);
#pragma unroll
                        for (uint32_t dst = 0; dst < CL; ++dst) st_cluster_v4(mapa(a, dst), w);
                    }
                }
                cl_sync(&ctl, cph, ct, P.err);
                bf16_land_to_operand(land(par), opnd, r, q);
                par ^= 1;
                signal_operand();
                wait_acc();
                if (epi_a) {
                    float v[16];
                    acc_sum(tmem, quarter, 0, nsplit(J_WO), v);
#pragma unroll
                    for (int rr = 0; rr < RB; ++rr) zs[rr * 64 + f_epi] += v[rr];
                }
                done_acc();
                // ------------------------------------- FFN
                bcast_slice_f32(zs, land(par), c, r, q);
                cl_sync(&ctl, cph, ct, P.err);
                norm_to_operand(land(par), P.g_ffn + l * D, P.eps, opnd, 0, r, q);
                par ^= 1;
                signal_operand();
                wait_acc();
                {   // SwiGLU: hidden chunk i = tiles 2i (W1) and 2i+1 (W3); pair a: i = 0, 2; pair b: i = 1
                    const int nh = nhid(c);
                    for (int i = epi_a ? 0 : 1; (epi_a || epi_b) && i < nh; i += 2) {
                        float h1[16], h3[16];
                        tmem_ld16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(2 * i * RB), h1);
                        tmem_ld16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)((2 * i + 1) * RB), h3);
                        uint8_t* chunk = hidb + i * CHUNK_BYTES;
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) {
                            const float a1 = h1[rr];
                            const float hv = a1 / (1.0f + expf(-a1)) * h3[rr];
                            *reinterpret_cast<bf16*>(chunk + swz(rr, f_epi >> 3) + (f_epi & 7) * 2) =
                                __float2bfloat16_rn(hv);
                        }
                    }
                }
                fence_before_sync();
                fence_proxy_async();
                bar_compute();
                if (ct == 0) mbar_arrive(&ctl.op_full);
                ++job;
                wait_acc();
                {   // W_2 partials for all 512 outputs -> the owner of each feature slice
                    for (int mt = epi_a ? 0 : 1; (epi_a || epi_b) && mt < 8; mt += 2) {
                        float v[16];
                        tmem_ld16(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(mt * RB), v);
                        const uint32_t a = smem_u32(land(par) + ((c * RB) * 64 + f_epi) * 4);
                        const uint32_t ra = mapa(a, (uint32_t)mt);
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) st_cluster_f32(ra + rr * 64 * 4, v[rr]);
                    }
                }
                done_acc();
                cl_sync(&ctl, cph, ct, P.err);
                {
                    const float* lp = reinterpret_cast<const float*>(land(par));
                    float4 acc = *reinterpret_cast<float4*>(zs + r * 64 + q * 4);
                    for (int src = 0; src < CL; ++src) {
                        const float4 pv = *reinterpret_cast<const float4*>(lp + (src * RB + r) * 64 + q * 4);
                        acc.x += pv.x; acc.y += pv.y; acc.z += pv.z; acc.w += pv.w;
                    }
                    *reinterpret_cast<float4*>(zs + r * 64 + q * 4) = acc;
                }
                par ^= 1;
                bar_compute();
            }
        }
        // state out (each CTA its own slice)
        if (valid)
            *reinterpret_cast<float4*>(P.s + (size_t)b * D + c * 64 + q * 4) =
                *reinterpret_cast<const float4*>(zs + r * 64 + q * 4);
    }
    fence_before_sync();
    __syncthreads();
    cluster_barrier_all();        // no peer still reads positions or writes this CTA's smem
    if (c == 0 && threadIdx.x < RB) {
        const int bb = (int)cluster_id_x() * RB + threadIdx.x;
        if (bb < P.B) P.pos_dec[bb] = pos_s[threadIdx.x] + P.nsteps;
    }
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace fz

// Launch nsteps fused transitions for all rows; false if the launch failed.
bool launch_dec_fused(const fz::FusedParams& p, cudaStream_t st) {
    if (!set_smem_once(reinterpret_cast<const void*>(fz::k_dec_fused), fz::SMEM_DYN))
        return false;
    const int nclusters = (p.B + fz::RB - 1) / fz::RB;
    fz::k_dec_fused<<<nclusters * fz::CL, fz::NT, fz::SMEM_DYN, st>>>(p);
    rlt_count_launch();
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace rlt
