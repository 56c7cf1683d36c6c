// C ABI of the RLT transition engine: weight-blob loading, state allocation
// and the host-side schedule of the encoder, the transition and the readout.
//
// The schedule follows the pages' execution procedures: the prompt is
// encoded token-parallel, then the decoder runs one transition per position,
// sequential within a row and batched across rows (jiphyeonjeon review
// "Recurrent Looped Transformer" §3.2, §5; greeksharifa "Recurrent Looped
// Transformer 요약 설명" §2.4, App. C.1, F.1-F.2); RLT-2 runs the positions of
// a chunk together (App. I.2).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/rlt.h"
#include "kernels.cuh"

// An NVTX range over each public call, so that a profiler's timeline shows
// which call the kernels and copies belong to (no-op without a profiler).
namespace {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace

static std::atomic<uint64_t> g_launches{0};
void rlt_count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace rlt {
// Programmatic dependent launch between consecutive kernels of a stream
// (and of a captured graph); RLT_PDL=0 launches them plainly.
bool pdl_enabled() {
    static const bool on = [] {
        const char* e = getenv("RLT_PDL");
        return !(e && strcmp(e, "0") == 0);
    }();
    return on;
}
// Function attributes are per device: each is set once per (device, kernel).
namespace {
std::mutex g_attr_mu;
std::set<std::tuple<int, const void*, int>> g_attr_done;   // (device, kernel, what)
int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return dev;
}
}  // namespace
void set_carveout_once(const void* kernel) {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (!g_attr_done.insert({current_device(), kernel, -1}).second) return;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        cudaGetLastError();        // a preference only: launching works without it
}
bool set_smem_once(const void* kernel, size_t bytes) {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    const auto key = std::make_tuple(current_device(), kernel, (int)bytes);
    if (g_attr_done.count(key)) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    g_attr_done.insert(key);
    return true;
}
int sm_count() {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, current_device()) !=
        cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}
template <typename T>
void launch_gemm(const T* A, int lda, const T* W, int ldw, float* C, int ldc, T* Ct, int ldct,
                 int M, int N, int K, int mode, cudaStream_t st);
}

using rlt::bf16;

// ============================================================================
// blob
// ============================================================================
namespace {

constexpr size_t kHeader = 256, kRecord = 64;

struct TensorSpec {
    std::string name;
    int d0, d1, ndim;
};

std::vector<TensorSpec> expected_manifest(const rlt_config& c) {
    std::vector<TensorSpec> v;
    const int d = c.d, f = c.ffn, V = c.vocab;
    auto mat = [&](const std::string& n, int a, int b) { v.push_back({n, a, b, 2}); };
    auto vec = [&](const std::string& n, int a) { v.push_back({n, a, 1, 1}); };
    mat("embed", V, d);
    if (c.variant != 0) vec("s_star", d);
    for (int l = 0; l < c.n_enc; ++l) {
        std::string p = "enc." + std::to_string(l) + ".";
        vec(p + "attn_norm", d);
        if (!c.tied) { mat(p + "wq", d, d); mat(p + "wk", d, d); mat(p + "wv", d, d); mat(p + "wo", d, d); }
        vec(p + "ffn_norm", d);
        if (!c.tied) { mat(p + "w1", f, d); mat(p + "w3", f, d); mat(p + "w2", d, f); }
    }
    if (c.n_dec > 0) {
        vec("mem_norm", d);
        for (int g = 0; g < c.groups; ++g) {
            mat("mem." + std::to_string(g) + ".wk", d, d);
            mat("mem." + std::to_string(g) + ".wv", d, d);
        }
    }
    if (c.variant != 0) {
        vec("merge.norm", d); mat("merge.wg", d, 2 * d); vec("merge.bg", d); mat("merge.ws", d, d);
    }
    for (int l = 0; l < c.n_dec; ++l) {
        std::string p = "dec." + std::to_string(l) + ".";
        vec(p + "swa_norm", d); mat(p + "wq", d, d); mat(p + "wk", d, d); mat(p + "wv", d, d);
        mat(p + "wo", d, d); vec(p + "x_norm", d); mat(p + "xq", d, d); mat(p + "xo", d, d);
        vec(p + "ffn_norm", d); mat(p + "w1", f, d); mat(p + "w3", f, d); mat(p + "w2", d, f);
    }
    vec("out_norm", d);
    mat("out", V, d);
    return v;
}

uint64_t blob_checksum(const uint8_t* p, size_t n) {
    uint64_t s = 0;
    size_t words = n / 8;
    for (size_t i = 0; i < words; ++i) {
        uint64_t w;
        memcpy(&w, p + 8 * i, 8);
        s += w * (2 * (uint64_t)i + 1);
    }
    return s;
}

float bf16_bits_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

struct ParsedBlob {
    rlt_config cfg;
    uint64_t checksum = 0;              // of the payload: identifies the weights
    std::vector<const uint8_t*> data;   // per manifest entry
};

int parse_blob(const void* blob, size_t nbytes, ParsedBlob* out) {
    if (!blob || nbytes < kHeader) return RLT_E_BLOB;
    const uint8_t* b = (const uint8_t*)blob;
    if (memcmp(b, "RLTB", 4) != 0) return RLT_E_BLOB;
    uint32_t ver;
    memcpy(&ver, b + 4, 4);
    if (ver != 1) return RLT_E_BLOB;
    uint32_t u[12];
    memcpy(u, b + 8, 48);
    rlt_config c;
    c.vocab = (int)u[0]; c.d = (int)u[1]; c.heads = (int)u[2]; c.n_enc = (int)u[3];
    c.n_dec = (int)u[4]; c.ffn = (int)u[5]; c.window = (int)u[6]; c.groups = (int)u[7];
    c.chunk = (int)u[8]; c.variant = (int)u[9]; c.tied = (int)u[10]; c.dtype = (int)u[11];
    memcpy(&c.alpha, b + 56, 8);
    memcpy(&c.eps, b + 64, 8);
    memcpy(&c.rope_base, b + 72, 8);
    uint64_t nt, nb, ck;
    memcpy(&nt, b + 88, 8);
    memcpy(&nb, b + 96, 8);
    memcpy(&ck, b + 104, 8);
    if (nb > nbytes - kHeader) return RLT_E_BLOB;
    const uint8_t* pay = b + kHeader;
    if (blob_checksum(pay, nb) != ck) return RLT_E_BLOB;
    if (c.dtype != RLT_DTYPE_F32 && c.dtype != RLT_DTYPE_BF16) return RLT_E_BLOB;
    // sizes far above any model this library runs, so that a malformed header
    // can neither overflow the manifest's int sizes nor make it huge
    if (c.vocab > (1 << 24) || c.d > (1 << 16) || c.ffn > (1 << 20) || c.n_enc > 4096 ||
        c.n_dec > 4096 || c.window > (1 << 24) || c.chunk > (1 << 24))
        return RLT_E_BLOB;
    if (c.vocab <= 0 || c.d <= 0 || c.heads <= 0 || c.d % c.heads || c.n_enc < 0 ||
        c.n_dec < 0 || c.ffn <= 0 || c.window < 1 || c.chunk < 1 || c.variant < 0 ||
        c.variant > 2 || (c.variant != 2 && c.chunk != 1) ||
        (c.groups != 1 && c.groups != c.n_dec) || c.groups < 1 ||
        (c.tied && c.n_enc != c.n_dec) || !(c.eps > 0) || !(c.rope_base > 0))
        return RLT_E_BLOB;
    std::vector<TensorSpec> man = expected_manifest(c);
    if (nt != man.size()) return RLT_E_BLOB;
    const size_t elt = c.dtype == RLT_DTYPE_BF16 ? 2 : 4;
    size_t off = 0;
    out->data.clear();
    for (const TensorSpec& s : man) {
        if (off + kRecord > nb) return RLT_E_BLOB;
        char name[49] = {0};
        memcpy(name, pay + off, 48);
        uint32_t r[4];
        memcpy(r, pay + off + 48, 16);
        if (s.name != name || (int)r[0] != s.ndim || (int)r[1] != c.dtype || (int)r[2] != s.d0 ||
            (int)r[3] != s.d1)
            return RLT_E_BLOB;
        off += kRecord;
        size_t bytes = (size_t)s.d0 * s.d1 * elt;
        if (off + bytes > nb) return RLT_E_BLOB;
        out->data.push_back(pay + off);
        off += bytes + ((64 - bytes % 64) % 64);
    }
    out->cfg = c;
    out->checksum = ck;
    return RLT_OK;
}

}  // namespace

// ============================================================================
// model
// ============================================================================
struct EncLayerW {
    float *attn_norm, *ffn_norm;
    void *wqkv, *wo, *w13, *w2;
};
struct DecLayerW {
    float *swa_norm, *x_norm, *ffn_norm;
    void *wqkv, *wo, *xq, *xo, *w13, *w2;
};

struct rlt_model {
    rlt_config cfg;
    uint64_t checksum = 0;          // the blob payload's checksum (the model's identity)
    int device = 0;
    int dh = 0, fpad = 0;
    size_t elt = 4;
    void* arena = nullptr;
    size_t arena_bytes = 0;
    void* embed = nullptr;
    float* s_star = nullptr;
    std::vector<EncLayerW> enc;
    float* mem_norm = nullptr;
    std::vector<void*> wmem;        // per group [2d][d]: K rows then V rows
    float *merge_norm = nullptr, *bg = nullptr;
    void* wgs = nullptr;
    std::vector<DecLayerW> dec;
    float* out_norm = nullptr;
    void* wout = nullptr;
};

namespace {

struct Arena {
    std::vector<uint8_t> host;
    size_t take(size_t bytes) {
        size_t off = (host.size() + 255) / 256 * 256;
        host.resize(off + bytes, 0);
        return off;
    }
};

// copy a stored matrix [rows][cols] into arena rows [row0..] of a [*, ld] matrix
void put_mat(Arena& a, size_t off, size_t elt, const uint8_t* src, int rows, int cols, int ld,
             int row0) {
    for (int r = 0; r < rows; ++r)
        memcpy(a.host.data() + off + ((size_t)(row0 + r) * ld) * elt, src + (size_t)r * cols * elt,
               (size_t)cols * elt);
}

void put_vec_f32(Arena& a, size_t off, size_t elt, const uint8_t* src, int n) {
    float* dst = (float*)(a.host.data() + off);
    for (int i = 0; i < n; ++i) {
        if (elt == 2) {
            uint16_t h;
            memcpy(&h, src + 2 * i, 2);
            dst[i] = bf16_bits_to_float(h);
        } else {
            memcpy(dst + i, src + 4 * i, 4);
        }
    }
}

}  // namespace

static int dev_err(cudaError_t e) {
    if (e == cudaErrorMemoryAllocation) return RLT_E_OOM;
    return e == cudaSuccess ? RLT_OK : RLT_E_DEVICE;
}

extern "C" int rlt_create(const void* blob, size_t nbytes, int device, rlt_model** out) {
    if (!out) return RLT_E_ARG;
    *out = nullptr;
    ParsedBlob pb;
    int rc = parse_blob(blob, nbytes, &pb);
    if (rc) return rc;
    const rlt_config& c = pb.cfg;
    const int dh = c.d / c.heads;
    if (dh != 16 && dh != 32 && dh != 64 && dh != 128) return RLT_E_UNSUPPORTED;
    if (c.d > 2048) return RLT_E_UNSUPPORTED;      // row kernels: one thread per 4 features
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        return RLT_E_DEVICE;
    }
    if (cudaSetDevice(device) != cudaSuccess) return RLT_E_DEVICE;

    rlt_model* m = new rlt_model();
    m->cfg = c;
    m->checksum = pb.checksum;
    m->device = device;
    m->dh = dh;
    m->fpad = (c.ffn + 63) / 64 * 64;
    m->elt = c.dtype == RLT_DTYPE_BF16 ? 2 : 4;
    const size_t elt = m->elt;
    const int d = c.d, fp = m->fpad;

    // lay the weights out in one arena: fused [3d][d] QKV, [2 fpad][d] W1;W3
    // (zero rows past ffn), [d][fpad] W2 (zero columns past ffn)
    Arena a;
    std::vector<TensorSpec> man = expected_manifest(c);
    auto idx = [&](const std::string& n) {
        for (size_t i = 0; i < man.size(); ++i)
            if (man[i].name == n) return (int)i;
        return -1;
    };
    auto src = [&](const std::string& n) { return pb.data[idx(n)]; };
    std::vector<std::pair<size_t, void**>> fixups;
    std::vector<std::pair<size_t, float**>> ffix;
    auto mat_plain = [&](const std::string& n, int rows, int cols, void** dst) {
        size_t off = a.take((size_t)rows * cols * elt);
        put_mat(a, off, elt, src(n), rows, cols, cols, 0);
        fixups.push_back({off, dst});
    };
    auto vecf = [&](const std::string& n, float** dst) {
        size_t off = a.take((size_t)d * 4);
        put_vec_f32(a, off, elt, src(n), d);
        ffix.push_back({off, dst});
    };
    auto qkv = [&](const std::string& p, void** dst) {
        size_t off = a.take((size_t)3 * d * d * elt);
        put_mat(a, off, elt, src(p + "wq"), d, d, d, 0);
        put_mat(a, off, elt, src(p + "wk"), d, d, d, d);
        put_mat(a, off, elt, src(p + "wv"), d, d, d, 2 * d);
        fixups.push_back({off, dst});
    };
    // W1 and W3 interleaved in blocks of 64 rows (w13_gate_col), so that a
    // 128-column output tile holds 64 gates and their up projections
    auto put_w13 = [&](Arena& ar, size_t o13, const uint8_t* w1, const uint8_t* w3) {
        for (int r = 0; r < c.ffn; ++r) {
            const int gr = rlt::w13_gate_col(r);
            put_mat(ar, o13, elt, w1 + (size_t)r * d * elt, 1, d, d, gr);
            put_mat(ar, o13, elt, w3 + (size_t)r * d * elt, 1, d, d, gr + rlt::kW13Block);
        }
    };
    auto ffn = [&](const std::string& p, void** w13, void** w2) {
        size_t o13 = a.take((size_t)2 * fp * d * elt);
        put_w13(a, o13, src(p + "w1"), src(p + "w3"));
        fixups.push_back({o13, w13});
        size_t o2 = a.take((size_t)d * fp * elt);
        put_mat(a, o2, elt, src(p + "w2"), d, c.ffn, fp, 0);
        fixups.push_back({o2, w2});
    };

    m->enc.resize(c.n_enc);
    m->dec.resize(c.n_dec);
    mat_plain("embed", c.vocab, d, &m->embed);
    if (c.variant != 0) vecf("s_star", &m->s_star);
    // decoder weights kind by kind: each kind is one [L_D * rows][cols] matrix
    // (every per-layer size is a multiple of the 256-byte arena step)
    auto dec_p = [&](int l) { return "dec." + std::to_string(l) + "."; };
    for (int l = 0; l < c.n_dec; ++l) vecf(dec_p(l) + "swa_norm", &m->dec[l].swa_norm);
    for (int l = 0; l < c.n_dec; ++l) vecf(dec_p(l) + "x_norm", &m->dec[l].x_norm);
    for (int l = 0; l < c.n_dec; ++l) vecf(dec_p(l) + "ffn_norm", &m->dec[l].ffn_norm);
    for (int l = 0; l < c.n_dec; ++l) qkv(dec_p(l), &m->dec[l].wqkv);
    for (int l = 0; l < c.n_dec; ++l) mat_plain(dec_p(l) + "wo", d, d, &m->dec[l].wo);
    for (int l = 0; l < c.n_dec; ++l) mat_plain(dec_p(l) + "xq", d, d, &m->dec[l].xq);
    for (int l = 0; l < c.n_dec; ++l) mat_plain(dec_p(l) + "xo", d, d, &m->dec[l].xo);
    {
        std::vector<void*> w2s(c.n_dec);
        for (int l = 0; l < c.n_dec; ++l) {
            size_t o13 = a.take((size_t)2 * fp * d * elt);
            put_w13(a, o13, src(dec_p(l) + "w1"), src(dec_p(l) + "w3"));
            fixups.push_back({o13, &m->dec[l].w13});
        }
        for (int l = 0; l < c.n_dec; ++l) {
            size_t o2 = a.take((size_t)d * fp * elt);
            put_mat(a, o2, elt, src(dec_p(l) + "w2"), d, c.ffn, fp, 0);
            fixups.push_back({o2, &m->dec[l].w2});
        }
    }
    for (int l = 0; l < c.n_enc; ++l) {
        std::string p = "enc." + std::to_string(l) + ".";
        EncLayerW& L = m->enc[l];
        vecf(p + "attn_norm", &L.attn_norm);
        vecf(p + "ffn_norm", &L.ffn_norm);
        if (!c.tied) {
            qkv(p, &L.wqkv);
            mat_plain(p + "wo", d, d, &L.wo);
            ffn(p, &L.w13, &L.w2);
        }
    }
    if (c.n_dec > 0) {
        vecf("mem_norm", &m->mem_norm);
        m->wmem.resize(c.groups);
        for (int g = 0; g < c.groups; ++g) {
            std::string p = "mem." + std::to_string(g) + ".";
            size_t off = a.take((size_t)2 * d * d * elt);
            put_mat(a, off, elt, src(p + "wk"), d, d, d, 0);
            put_mat(a, off, elt, src(p + "wv"), d, d, d, d);
            fixups.push_back({off, &m->wmem[g]});
        }
    }
    if (c.variant != 0) {
        vecf("merge.norm", &m->merge_norm);
        vecf("merge.bg", &m->bg);
        // both merge projections as one [2d][2d] matrix over [e_t; r]: rows
        // 0..d-1 are W_g, rows d..2d-1 are [0 | W_s] (one GEMM launch)
        size_t og = a.take((size_t)4 * d * d * elt);
        put_mat(a, og, elt, src("merge.wg"), d, 2 * d, 2 * d, 0);
        const uint8_t* wsrc = src("merge.ws");
        for (int r = 0; r < d; ++r)
            memcpy(a.host.data() + og + ((size_t)(d + r) * 2 * d + d) * elt,
                   wsrc + (size_t)r * d * elt, (size_t)d * elt);
        fixups.push_back({og, &m->wgs});
    }
    vecf("out_norm", &m->out_norm);
    mat_plain("out", c.vocab, d, &m->wout);

    m->arena_bytes = a.host.size();
    cudaError_t e = cudaMalloc(&m->arena, m->arena_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        delete m;
        return dev_err(e);
    }
    e = cudaMemcpy(m->arena, a.host.data(), m->arena_bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(m->arena);
        delete m;
        return RLT_E_DEVICE;
    }
    uint8_t* base = (uint8_t*)m->arena;
    for (auto& fx : fixups) *fx.second = base + fx.first;
    for (auto& fx : ffix) *fx.second = (float*)(base + fx.first);
    if (c.tied) {
        for (int l = 0; l < c.n_enc; ++l) {
            m->enc[l].wqkv = m->dec[l].wqkv;
            m->enc[l].wo = m->dec[l].wo;
            m->enc[l].w13 = m->dec[l].w13;
            m->enc[l].w2 = m->dec[l].w2;
        }
    }
    *out = m;
    return RLT_OK;
}

extern "C" void rlt_destroy(rlt_model* m) {
    if (!m) return;
    cudaSetDevice(m->device);
    cudaFree(m->arena);
    delete m;
}

extern "C" int rlt_model_config(const rlt_model* m, rlt_config* out) {
    if (!m || !out) return RLT_E_ARG;
    *out = m->cfg;
    return RLT_OK;
}

// ============================================================================
// state
// ============================================================================
struct rlt_state {
    rlt_model* m = nullptr;
    int B = 0, T_cap = 0;
    int n_enc_blk = 1, n_dec_blk = 1;    // positions per row in one encoder / decoder pass
    float *s = nullptr, *Rr = nullptr, *e = nullptr;
    void *enc = nullptr, *mem = nullptr, *ring = nullptr;
    size_t enc_row = 0, mem_row = 0, ring_row = 0;   // elements per row
    int32_t *pos_enc = nullptr, *pos_dec = nullptr;
    std::vector<int32_t> h_pos_enc, h_pos_dec;
    float *rope_cs = nullptr, *rope_sn = nullptr;
    int* err = nullptr;
    // scratch (rows = B * max block)
    float *X = nullptr, *QKV = nullptr, *Q = nullptr, *H13 = nullptr, *G = nullptr, *S = nullptr;
    void *Y = nullptr, *Hd = nullptr, *A = nullptr, *Kc = nullptr, *Vc = nullptr;
    int32_t* tok = nullptr;
    float* logits = nullptr;
    int32_t* ids = nullptr;
    int32_t* rows = nullptr;
    float* replay_lp = nullptr;     // rlt_replay_logprobs: [B][T_cap], allocated on first use
    int32_t* replay_tok = nullptr;
    float* P = nullptr;             // split-K partial slabs of the transition's projections
    size_t p_cols = 0;              // columns of one slab row (the widest projection)
    int p_slabs = 1;                // slabs allocated
    std::vector<void*> allocs;
    size_t bytes = 0;
    // live timing (rlt_profile_*)
    bool prof = false;
    int prof_level = 0;               // 2: also time each attention launch inside the graphs
    // a record holds its events until queried, or (events owned by a graph)
    // the elapsed time read right after the replay
    struct ProfRec { int cls; cudaEvent_t a, b; double bytes; float ms; int layer; };
    std::vector<ProfRec> prof_recs;
    std::vector<cudaEvent_t> prof_pool;
    // event pairs captured into a graph (cudaEventRecordExternal nodes), with
    // the index of the block they bracket
    struct CapRec { int cls; cudaEvent_t a, b; int block; int layer; int b0, nb; };
    bool prof_capture = false;
    int prof_block = 0;
    int prof_b0 = 0, prof_nb = 0;     // rows of the transition block being issued
    std::vector<CapRec> cap_recs;
    // replayable transition blocks, per positions-per-block n; graphs_prof
    // carries event nodes around the attention launches (profiling level 2)
    struct Graph { cudaGraphExec_t exec; uint64_t launches; std::vector<CapRec> caps; };
    std::map<int, Graph> graphs, graphs_prof;
    // streams of the row groups after the first inside a captured graph
    std::vector<cudaStream_t> aux;
};

static cudaEvent_t prof_event(rlt_state* s) {
    cudaEvent_t e = nullptr;
    if (!s->prof_pool.empty()) {
        e = s->prof_pool.back();
        s->prof_pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}
// Bracket a launch sequence with events on `st` when profiling is on.
struct ProfScope {
    rlt_state* s;
    int cls;
    cudaStream_t st;
    double bytes;
    int layer;
    cudaEvent_t a = nullptr;
    bool cap = false;
    ProfScope(rlt_state* s_, int c, cudaStream_t st_, double b, int l = -1)
        : s(s_), cls(c), st(st_), bytes(b), layer(l) {
        if (s->prof_capture) {          // becomes an event node of the graph being captured
            if (cudaEventCreate(&a) != cudaSuccess) {
                cudaGetLastError();
                a = nullptr;
                return;
            }
            cap = true;
            cudaEventRecordWithFlags(a, st, cudaEventRecordExternal);
        } else if (s->prof && (a = prof_event(s))) {
            cudaEventRecord(a, st);
        }
    }
    ~ProfScope() {
        if (!a) return;
        if (cap) {
            cudaEvent_t b = nullptr;
            if (cudaEventCreate(&b) != cudaSuccess) {
                cudaGetLastError();
                cudaEventDestroy(a);
                return;
            }
            cudaEventRecordWithFlags(b, st, cudaEventRecordExternal);
            s->cap_recs.push_back({cls, a, b, s->prof_block, layer, s->prof_b0, s->prof_nb});
            return;
        }
        cudaEvent_t b = prof_event(s);
        if (!b) return;
        cudaEventRecord(b, st);
        s->prof_recs.push_back({cls, a, b, bytes, -1.f, layer});
    }
};

static int salloc(rlt_state* s, void** p, size_t bytes) {
    if (bytes == 0) bytes = 256;
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return dev_err(e);
    }
    s->allocs.push_back(*p);
    s->bytes += bytes;
    return RLT_OK;
}

extern "C" void rlt_state_destroy(rlt_state* s) {
    if (!s) return;
    cudaSetDevice(s->m->device);
    cudaDeviceSynchronize();
    for (auto& r : s->prof_recs) {
        if (r.a) cudaEventDestroy(r.a);
        if (r.b) cudaEventDestroy(r.b);
    }
    for (cudaEvent_t e : s->prof_pool) cudaEventDestroy(e);
    for (auto* gm : {&s->graphs, &s->graphs_prof})
        for (auto& g : *gm) {
            cudaGraphExecDestroy(g.second.exec);
            for (auto& c : g.second.caps) {
                cudaEventDestroy(c.a);
                cudaEventDestroy(c.b);
            }
        }
    for (cudaStream_t a : s->aux) cudaStreamDestroy(a);
    for (void* p : s->allocs) cudaFree(p);
    delete s;
}

static int max_dec_splits(const rlt_config& c, int fp);

static size_t max_rows_per_call() {
    const char* v = getenv("RLT_MAX_ROWS");
    long x = v ? atol(v) : 65536;
    return (size_t)std::max(256L, x);
}

extern "C" int rlt_state_create(rlt_model* m, int batch, int max_len, rlt_state** out) {
    if (!m || !out || batch <= 0 || max_len <= 0) return RLT_E_ARG;
    *out = nullptr;
    if (cudaSetDevice(m->device) != cudaSuccess) return RLT_E_DEVICE;
    const rlt_config& c = m->cfg;
    {   // every allocation below (caches, rings, scratch, split-K slabs,
        // logits) is at most this product of the caller's sizes: refuse the
        // sizes whose byte counts could wrap around
        using u128 = unsigned __int128;
        const u128 bound = (u128)batch *
                           (u128)((size_t)max_len + (size_t)c.window + (size_t)c.chunk + 16) *
                           (u128)(3 * (size_t)c.d + 2 * (size_t)m->fpad + (size_t)c.vocab) * 4 *
                           (u128)(2 * ((size_t)c.n_enc + c.n_dec + c.groups) + 8);
        if (bound > ((u128)1 << 60)) return RLT_E_OOM;
    }
    rlt_state* s = new rlt_state();
    s->m = m;
    s->B = batch;
    s->T_cap = max_len;
    const size_t elt = m->elt, d = c.d, dh = m->dh, h = c.heads, B = batch, T = max_len;
    const size_t slots = (size_t)std::max(0, c.window - 1);
    size_t maxr = max_rows_per_call();
    s->n_enc_blk = (int)std::max<size_t>(1, std::min<size_t>(T, maxr / B));
    s->n_dec_blk = c.variant == 2 ? c.chunk : (c.variant == 0 ? std::min(s->n_enc_blk, 16) : 1);
    const size_t R = B * (size_t)std::max(s->n_enc_blk, s->n_dec_blk);
    s->enc_row = (size_t)c.n_enc * 2 * h * T * dh;
    s->mem_row = (size_t)(c.n_dec > 0 ? c.groups : 0) * 2 * h * T * dh;
    s->ring_row = (size_t)c.n_dec * 2 * h * slots * dh;
    int rc = RLT_OK;
    auto take = [&](void** p, size_t bytes) {
        if (rc == RLT_OK) rc = salloc(s, p, bytes);
    };
    const size_t fp = m->fpad;
    take((void**)&s->s, B * d * 4);
    take((void**)&s->Rr, B * d * 4);
    take((void**)&s->e, B * T * d * 4);
    take(&s->enc, B * s->enc_row * elt);
    take(&s->mem, B * s->mem_row * elt);
    take(&s->ring, B * s->ring_row * elt);
    take((void**)&s->pos_enc, B * 4);
    take((void**)&s->pos_dec, B * 4);
    take((void**)&s->rope_cs, (T + 1) * (dh / 2) * 4);
    take((void**)&s->rope_sn, (T + 1) * (dh / 2) * 4);
    take((void**)&s->err, 4);
    take((void**)&s->X, R * d * 4);
    take((void**)&s->QKV, R * 3 * d * 4);
    take((void**)&s->Q, R * d * 4);
    take((void**)&s->H13, R * 2 * fp * 4);
    take((void**)&s->G, R * d * 4);
    take((void**)&s->S, R * d * 4);
    take(&s->Y, R * std::max(2 * d, fp) * elt);
    take(&s->Hd, R * fp * elt);
    take(&s->A, R * d * elt);
    take(&s->Kc, R * d * elt);
    take(&s->Vc, R * d * elt);
    take((void**)&s->tok, R * 4);
    take((void**)&s->logits, B * (size_t)c.vocab * 4);
    take((void**)&s->ids, 2 * B * 4);
    take((void**)&s->rows, B * 4);
    {   // split-K slabs for the transition: widest projection x most splits
        const size_t Rd = B * (size_t)s->n_dec_blk;
        s->p_cols = std::max<size_t>(3 * d, 2 * fp);
        s->p_slabs = max_dec_splits(c, (int)fp);
        take((void**)&s->P, (size_t)s->p_slabs * Rd * s->p_cols * 4);
    }
    if (rc != RLT_OK) {
        rlt_state_destroy(s);
        return rc;
    }
    // RoPE table: angle p * base^(-2i/dh) for p = 0..T, computed in double
    std::vector<float> cs((T + 1) * (dh / 2)), sn((T + 1) * (dh / 2));
    for (size_t p = 0; p <= T; ++p)
        for (size_t i = 0; i < dh / 2; ++i) {
            double ang = (double)p * std::pow(c.rope_base, -2.0 * (double)i / (double)dh);
            cs[p * (dh / 2) + i] = (float)std::cos(ang);
            sn[p * (dh / 2) + i] = (float)std::sin(ang);
        }
    cudaError_t e1 = cudaMemcpy(s->rope_cs, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice);
    cudaError_t e2 = cudaMemcpy(s->rope_sn, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice);
    cudaError_t e3 = cudaMemset(s->err, 0, 4);
    if (e1 || e2 || e3) {
        rlt_state_destroy(s);
        return RLT_E_DEVICE;
    }
    s->h_pos_enc.assign(B, 0);
    s->h_pos_dec.assign(B, 0);
    rlt::launch_reset_rows(nullptr, batch, m->s_star, s->s, s->Rr, s->pos_enc, s->pos_dec, c.d,
                           0);
    if (cudaDeviceSynchronize() != cudaSuccess) {
        rlt_state_destroy(s);
        return RLT_E_DEVICE;
    }
    *out = s;
    return RLT_OK;
}

extern "C" int rlt_state_bytes(const rlt_state* s, size_t* per_row_state, size_t* total) {
    if (!s) return RLT_E_ARG;
    const rlt_config& c = s->m->cfg;
    if (per_row_state)
        *per_row_state = (s->enc_row + s->mem_row + s->ring_row) * s->m->elt + (size_t)c.d * 4;
    if (total) *total = s->bytes;
    return RLT_OK;
}

// ============================================================================
// helpers
// ============================================================================
static bool is_device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

static int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? RLT_OK : RLT_E_DEVICE;
}

static rlt::RopeTab rope_of(rlt_state* s) {
    return rlt::RopeTab{s->rope_cs, s->rope_sn, s->m->dh / 2, s->T_cap};
}

// ============================================================================
// algorithmic bytes of one launch (what the computation must move at least;
// weights excluded unless they cannot stay on chip)
// ============================================================================
static double kv_bytes(const rlt_state* s) { return 2.0 * s->m->cfg.d * (double)s->m->elt; }

// (rows b0 .. b0+nb-1; all rows by default)
static double xattn_bytes(const rlt_state* s, int n, int b0 = 0, int nb = -1) {
    const double d = s->m->cfg.d, elt = (double)s->m->elt;
    double by = 0;
    for (int b = b0; b < (nb < 0 ? s->B : b0 + nb); ++b)
        by += (s->h_pos_dec[b] + n) * kv_bytes(s) + n * (d * 4 + d * elt);
    return by;
}
static double swa_bytes(const rlt_state* s, int n, int b0 = 0, int nb = -1) {
    const double d = s->m->cfg.d, elt = (double)s->m->elt;
    const int slots = std::max(0, s->m->cfg.window - 1);
    double by = 0;
    for (int b = b0; b < (nb < 0 ? s->B : b0 + nb); ++b)
        by += std::min(s->h_pos_dec[b], slots) * kv_bytes(s) + n * (kv_bytes(s) + d * 4 + d * elt);
    return by;
}
static double decoder_weight_bytes(const rlt_model* m) {
    const double d = m->cfg.d, f = m->cfg.ffn;
    return (double)m->elt * (m->cfg.n_dec * (6 * d * d + 3 * d * f) + (m->cfg.variant ? 3 * d * d : 0));
}
static double step_bytes(const rlt_state* s, int n) {    // one whole transition block
    const rlt_config& c = s->m->cfg;
    const int slots = std::max(0, c.window - 1);
    double by = 0;
    for (int b = 0; b < s->B; ++b) {
        const int pd = s->h_pos_dec[b];
        by += c.n_dec * ((pd + n) * kv_bytes(s) + std::min(pd, slots) * kv_bytes(s) +
                         std::min(n, slots) * kv_bytes(s));
        by += n * c.d * 4.0 + 2.0 * c.d * 4.0;            // e_t in, s in and out
    }
    // weights re-stream from HBM each step once they exceed what L2 can hold
    if (decoder_weight_bytes(s->m) > 64e6) by += decoder_weight_bytes(s->m);
    return by;
}
static double enc_bytes(const rlt_state* s, int n) {     // one encoder block
    const rlt_config& c = s->m->cfg;
    double by = 0;
    for (int b = 0; b < s->B; ++b) {
        const int p0 = s->h_pos_enc[b];
        // cache and memory written for n positions; cached keys/values re-read
        by += (c.n_enc + (c.n_dec ? c.groups : 0)) * n * kv_bytes(s) +
              c.n_enc * (double)p0 * kv_bytes(s) + n * (4.0 + c.d * 4.0);
    }
    return by;
}

// Split-K factor of a transition projection (N outputs, K inputs): as many
// CTAs as fit one wave on the machine when M = 256 rows (a second wave costs
// more than the longer K run), a function of N and K only (never of the
// batch), at least two 64-wide K-chunks per split.  Products of 4 MB of
// weights or more (the d = 2048 model, whose batches are tens of rows) stream
// their weights: two CTAs per SM over one 128-row tile keep enough weight
// bytes in flight.  1 for fp32 models.
static int dec_splits_for(const rlt_config& c, int N, int K) {
    if (c.dtype != RLT_DTYPE_BF16 || K % 64) return 1;
    const int ntile = (N + 63) / 64;
    const int tiles = 2 * ntile;                      // output tiles at M = 256
    const int nk = K / 64;
    const bool heavy = 2.0 * N * K >= 4e6;
    int want = heavy ? std::max(1, 2 * 148 / ntile) : std::max(1, 148 / tiles);
    want = std::min({want, std::max(1, nk / 2), 8});      // consumers sum at most 8 slabs
    const int cps = (nk + want - 1) / want;
    return (nk + cps - 1) / cps;
}
static int dec_splits(const rlt_state* s, int N, int K) {
    return std::min(s->p_slabs, dec_splits_for(s->m->cfg, N, K));
}
// the most slabs any transition projection of this model uses
static int max_dec_splits(const rlt_config& c, int fp) {
    const int d = c.d;
    const int shapes[6][2] = {{3 * d, d}, {d, d}, {2 * fp, d}, {d, fp}, {2 * d, 2 * d}, {d, d}};
    int m = 1;
    for (auto& sh : shapes) m = std::max(m, dec_splits_for(c, sh[0], sh[1]));
    return m;
}

// ============================================================================
// encoder
// ============================================================================
// The encoder's causal attention runs on the tensor cores (q and the
// probabilities enter the MMAs as bf16) with the short kernel whenever
// d_h = 64 and no row's prefix passes 256 keys, and with the key-tiled
// kernel (d_h = 128, longer prefixes) for encode calls of at least this many
// new positions per row (prompts); shorter calls there (generation steps)
// stream the keys on the CUDA cores with q and p in fp32: the key-tiled
// kernel would walk every key tile twice for a mostly empty query tile.
static constexpr int kEncTcMinPositions = 16;

template <typename T>
static void encode_block(rlt_state* s, const int32_t* tok, int n, cudaStream_t st,
                         bool tc_attn) {
    using namespace rlt;
    rlt_model* m = s->m;
    const rlt_config& c = m->cfg;
    const int B = s->B, d = c.d, h = c.heads, dh = m->dh, fp = m->fpad, R = B * n;
    const float eps = (float)c.eps;
    T* Y = (T*)s->Y;
    T* A = (T*)s->A;
    T* Hd = (T*)s->Hd;
    T* enc = (T*)s->enc;
    const size_t layer_enc = (size_t)2 * h * s->T_cap * dh;
    launch_check_positions(s->pos_enc, s->pos_dec, B, n, s->T_cap, true, s->err, st);
    launch_embed<T>((const T*)m->embed, tok, s->X, R, d, c.vocab, s->err, st);
    int max_keys = 0;                        // longest cache prefix any row attends to
    for (int b = 0; b < B; ++b) max_keys = std::max(max_keys, s->h_pos_enc[b] + n);
    for (int l = 0; l < c.n_enc; ++l) {
        const EncLayerW& L = m->enc[l];
        launch_rmsnorm<T>(s->X, d, L.attn_norm, Y, d, R, d, eps, st);
        // many rows: RoPE and the cache scatter in the q|k|v GEMM's epilogue
        bool qkv_done = false;
        if constexpr (std::is_same<T, bf16>::value)
            qkv_done = launch_gemm_rope_scatter(
                Y, d, (const bf16*)L.wqkv, d, R, 3 * d, d,
                RopeScatter{s->Q, enc + l * layer_enc, s->enc_row, s->T_cap, s->pos_enc,
                            rope_of(s), n, dh, d, 0},
                st);
        if (!qkv_done) {
            launch_gemm<T>(Y, d, (const T*)L.wqkv, d, s->QKV, 3 * d, nullptr, 0, R, 3 * d, d,
                           kStoreF32, st);
            launch_qkv_enc<T>(s->QKV, s->pos_enc, rope_of(s), s->Q, enc + l * layer_enc,
                              s->enc_row, s->T_cap, B, n, h, dh, st);
        }
        bool attn_done = false;
        if constexpr (std::is_same<T, bf16>::value)
            attn_done = (tc_attn || (dh == 64 && max_keys <= 256)) && fast_attn_enabled() &&
                        launch_attn_enc_tc(s->Q, enc + l * layer_enc, s->enc_row, s->T_cap,
                                           s->pos_enc, A, B, n, h, dh, max_keys, s->err, st);
        if constexpr (std::is_same<T, bf16>::value)
            if (!attn_done && n == 1)
                attn_done = launch_attn_enc_step(s->Q, enc + l * layer_enc, s->enc_row, s->T_cap,
                                                 s->pos_enc, A, B, h, dh, st);
        if (!attn_done)
            launch_attn_enc<T>(s->Q, enc + l * layer_enc, s->enc_row, s->T_cap, s->pos_enc, A, B,
                               n, h, dh, st);
        launch_gemm<T>(A, d, (const T*)L.wo, d, s->X, d, nullptr, 0, R, d, d, kAddF32, st);
        launch_rmsnorm<T>(s->X, d, L.ffn_norm, Y, d, R, d, eps, st);
        bool ffn_done = false;
        if constexpr (std::is_same<T, bf16>::value)
            ffn_done = launch_gemm_swiglu(Y, d, (const bf16*)L.w13, d, Hd, fp, R, 2 * fp, d, st);
        if (!ffn_done) {
            launch_gemm<T>(Y, d, (const T*)L.w13, d, s->H13, 2 * fp, nullptr, 0, R, 2 * fp, d,
                           kStoreF32, st);
            launch_swiglu<T>(s->H13, 1, 0, fp, Hd, R, st);
        }
        launch_gemm<T>(Hd, fp, (const T*)L.w2, fp, s->X, d, nullptr, 0, R, d, fp, kAddF32, st);
    }
    launch_copy_e(s->X, s->pos_enc, s->e, s->T_cap, B, n, d, st);
    if (c.n_dec > 0) {
        launch_rmsnorm<T>(s->X, d, m->mem_norm, Y, d, R, d, eps, st);
        const size_t layer_mem = (size_t)2 * h * s->T_cap * dh;
        for (int g = 0; g < c.groups; ++g) {
            T* mem_g = (T*)s->mem + g * layer_mem;
            bool kv_done = false;
            if constexpr (std::is_same<T, bf16>::value)
                kv_done = launch_gemm_rope_scatter(
                    Y, d, (const bf16*)m->wmem[g], d, R, 2 * d, d,
                    RopeScatter{nullptr, mem_g, s->mem_row, s->T_cap, s->pos_enc, rope_of(s), n,
                                dh, d, 1},
                    st);
            if (!kv_done) {
                launch_gemm<T>(Y, d, (const T*)m->wmem[g], d, s->QKV, 2 * d, nullptr, 0, R,
                               2 * d, d, kStoreF32, st);
                launch_mem_scatter<T>(s->QKV, s->pos_enc, rope_of(s), mem_g, s->mem_row,
                                      s->T_cap, B, n, h, dh, st);
            }
        }
    }
    launch_pos_add(s->pos_enc, B, n, st);
}

extern "C" int rlt_encode(rlt_state* s, const int32_t* tokens, int n, void* stream) {
    NvtxRange nvtx("rlt_encode");
    if (!s || !tokens || n < 0) return RLT_E_ARG;
    if (n == 0) return RLT_OK;
    rlt_model* m = s->m;
    if (cudaSetDevice(m->device) != cudaSuccess) return RLT_E_DEVICE;
    for (int b = 0; b < s->B; ++b)
        if (s->h_pos_enc[b] + n > s->T_cap) return RLT_E_CAPACITY;
    cudaStream_t st = (cudaStream_t)stream;
    const bool dev = is_device_ptr(tokens);
    if (!dev) {
        for (size_t i = 0; i < (size_t)s->B * n; ++i)
            if (tokens[i] < 0 || tokens[i] >= m->cfg.vocab) return RLT_E_ARG;
    }
    // rows of the caller's [B][n] array are split into blocks of n_enc_blk positions
    for (int j0 = 0; j0 < n; j0 += s->n_enc_blk) {
        int nb = std::min(s->n_enc_blk, n - j0);
        cudaError_t e = cudaMemcpy2DAsync(s->tok, (size_t)nb * 4, tokens + j0, (size_t)n * 4,
                                          (size_t)nb * 4, s->B,
                                          dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice,
                                          st);
        if (e != cudaSuccess) return RLT_E_DEVICE;
        {
            ProfScope ps(s, n == 1 ? RLT_PROF_ENC1 : RLT_PROF_ENC, st,
                         s->prof ? enc_bytes(s, nb) : 0.0);
            const bool tc = n >= kEncTcMinPositions;      // by the call, not the block
            if (m->cfg.dtype == RLT_DTYPE_BF16) encode_block<bf16>(s, s->tok, nb, st, tc);
            else encode_block<float>(s, s->tok, nb, st, tc);
        }
        int rc = launch_status();
        if (rc) return rc;
        // the next block's launch shapes (its longest key prefix) read the
        // host copy of the positions: advance it block by block
        for (int b = 0; b < s->B; ++b) s->h_pos_enc[b] += nb;
    }
    return RLT_OK;
}

// ============================================================================
// transition
// ============================================================================
// merged_in: the previous block already wrote this block's merge input (Y);
// fuse_out: end with the state hand-off fused with the next block's merge
// input (one position per row, RLT-1/2, inside a replayed run of blocks).
// b0, nb: the block runs rows b0 .. b0+nb-1 only (all rows by default).  A
// row range keeps its own part of every scratch buffer (rows b0*n.. at each
// buffer's widest pitch), so the ranges of one block can run concurrently.
template <typename T>
static void step_block(rlt_state* s, int n, cudaStream_t st, bool merged_in = false,
                       bool fuse_out = false, int b0 = 0, int nb = -1) {
    using namespace rlt;
    rlt_model* m = s->m;
    const rlt_config& c = m->cfg;
    const int B = nb < 0 ? s->B : nb, d = c.d, h = c.heads, dh = m->dh, fp = m->fpad,
              R = B * n;
    const float eps = (float)c.eps;
    const size_t row0 = (size_t)b0 * n;
    T* Y = (T*)s->Y + row0 * std::max(2 * d, fp);
    T* A = (T*)s->A + row0 * d;
    T* Hd = (T*)s->Hd + row0 * fp;
    T* Kc = (T*)s->Kc + row0 * d;
    T* Vc = (T*)s->Vc + row0 * d;
    float* z = s->X + row0 * d;
    float* Q = s->Q + row0 * d;
    int32_t* pos_dec = s->pos_dec + b0;
    const float* e = s->e + (size_t)b0 * s->T_cap * d;
    float* s_vec = s->s + (size_t)b0 * d;
    float* r_reg = s->Rr + (size_t)b0 * d;
    s->prof_b0 = b0;
    s->prof_nb = B;
    // Split-K partial slabs of each projection land in s->P; the kernel that
    // consumes the projection adds them in slab order (residual projections:
    // the next RMSNorm, or the state hand-off).
    float* P = s->P + row0 * s->p_cols;
    const size_t slab = (size_t)s->B * n * s->p_cols;
    auto gemm_p = [&](const T* Ain, int lda, const T* Wt, int N, int K, float* dst) {
        return launch_gemm_split<T>(Ain, lda, Wt, K, dst, N, R, N, K, dec_splits(s, N, K), slab,
                                    st);
    };
    // the merge kernel also applies the first decoder block's input RMSNorm
    const float* norm0 = c.n_dec > 0 ? m->dec[0].swa_norm : nullptr;
    launch_check_positions(s->pos_enc + b0, pos_dec, B, n, s->T_cap, false, s->err, st);
    if (c.variant == 0) {
        launch_merge_out<T>(e, s->T_cap, pos_dec, nullptr, 0, 0, nullptr, nullptr, 0, 0, d, 0.f,
                            z, norm0, Y, eps, B, n, d, st);
    } else {
        const float* fb = c.variant == 2 ? r_reg : s_vec;
        if (!merged_in)
            launch_merge_input<T>(e, s->T_cap, pos_dec, fb, m->merge_norm, Y, B, n, d, eps, st);
        // one GEMM for both projections: gate pre-activations in columns
        // 0..d-1 of the slabs, W_s r in columns d..2d-1
        const int nGS = gemm_p(Y, 2 * d, (const T*)m->wgs, 2 * d, 2 * d, P);
        launch_merge_out<T>(e, s->T_cap, pos_dec, P, nGS, slab, m->bg, P + d, nGS, slab, 2 * d,
                            (float)c.alpha, z, norm0, Y, eps, B, n, d, st);
    }
    const size_t layer_ring = (size_t)2 * h * std::max(0, c.window - 1) * dh;
    const size_t layer_mem = (size_t)2 * h * s->T_cap * dh;
    int nres = 0;                       // pending residual partial slabs in P
    for (int l = 0; l < c.n_dec; ++l) {
        const DecLayerW& L = m->dec[l];
        T* ring = (T*)s->ring + (size_t)b0 * s->ring_row + l * layer_ring;
        if (l > 0)
            launch_add_rmsnorm<T>(z, nres ? P : nullptr, nres, slab, L.swa_norm, Y, R, d, eps, st);
        int np = gemm_p(Y, d, (const T*)L.wqkv, 3 * d, d, P);
        {
            // bf16: the attention kernel forms q, k, v from the slabs and
            // updates the ring itself; otherwise scatter, attend, write
            ProfScope ps(s, RLT_PROF_SWA, st, s->prof ? swa_bytes(s, n, b0, B) : 0.0, l);
            bool done = false;
            if constexpr (std::is_same<T, bf16>::value)
                done = launch_attn_swa_proj(ProjIn{P, np, slab, 3 * d, rope_of(s)}, ring,
                                            s->ring_row, c.window, pos_dec, A, B, n, h, dh, st);
            if (!done) {
                launch_qkv_dec<T>(P, np, slab, pos_dec, rope_of(s), Q, Kc, Vc, B, n, h, dh, st);
                launch_attn_swa<T>(Q, Kc, Vc, ring, s->ring_row, c.window, pos_dec, A, B, n, h,
                                   dh, st);
                launch_ring_write<T>(Kc, Vc, pos_dec, ring, s->ring_row, c.window, B, n, h, dh,
                                     st);
            }
        }
        nres = gemm_p(A, d, (const T*)L.wo, d, d, P);
        launch_add_rmsnorm<T>(z, P, nres, slab, L.x_norm, Y, R, d, eps, st);
        np = gemm_p(Y, d, (const T*)L.xq, d, d, P);
        const T* mem =
            (const T*)s->mem + (size_t)b0 * s->mem_row + (c.groups > 1 ? l : 0) * layer_mem;
        {
            ProfScope ps(s, RLT_PROF_XATTN, st, s->prof ? xattn_bytes(s, n, b0, B) : 0.0, l);
            bool done = false;
            if constexpr (std::is_same<T, bf16>::value)
                done = launch_attn_cross_proj(ProjIn{P, np, slab, d, rope_of(s)}, mem, s->mem_row,
                                              s->T_cap, pos_dec, A, B, n, h, dh, st);
            if (!done) {
                launch_rope_q(P, np, slab, Q, pos_dec, rope_of(s), B, n, h, dh, st);
                launch_attn_cross<T>(Q, mem, s->mem_row, s->T_cap, pos_dec, A, B, n, h, dh, st);
            }
        }
        nres = gemm_p(A, d, (const T*)L.xo, d, d, P);
        launch_add_rmsnorm<T>(z, P, nres, slab, L.ffn_norm, Y, R, d, eps, st);
        // SwiGLU in the GEMM epilogue whenever W1;W3 is not split (64-wide
        // tiles hold 32 gates and their ups); a split product goes through
        // its slabs and the row kernel
        bool ffn_done = false;
        if constexpr (std::is_same<T, bf16>::value)
            ffn_done = (R >= 2048 || dec_splits(s, 2 * fp, d) == 1) &&
                       launch_gemm_swiglu(Y, d, (const bf16*)L.w13, d, Hd, fp, R, 2 * fp, d, st);
        if (!ffn_done) {
            np = gemm_p(Y, d, (const T*)L.w13, 2 * fp, d, P);
            launch_swiglu<T>(P, np, slab, fp, Hd, R, st);
        }
        nres = gemm_p(Hd, fp, (const T*)L.w2, d, fp, P);
    }
    if (fuse_out)
        launch_state_merge<T>(z, nres ? P : nullptr, nres, slab, s_vec,
                              c.variant == 2 ? r_reg : nullptr, pos_dec, c.chunk, e, s->T_cap,
                              m->merge_norm, Y, B, d, eps, st);
    else
        launch_set_state(z, nres ? P : nullptr, nres, slab, s_vec,
                         c.variant == 2 ? r_reg : nullptr, pos_dec, c.chunk, B, n, d,
                         /*bump=*/true, st);
}

static int run_block(rlt_state* s, int n, cudaStream_t st) {
    for (int b = 0; b < s->B; ++b) {
        if (s->h_pos_dec[b] + n > s->h_pos_enc[b]) return RLT_E_ORDER;
        if (s->h_pos_dec[b] + n > s->T_cap) return RLT_E_CAPACITY;
    }
    {
        ProfScope ps(s, RLT_PROF_STEP, st, s->prof ? step_bytes(s, n) : 0.0);
        if (s->m->cfg.dtype == RLT_DTYPE_BF16) step_block<bf16>(s, n, st);
        else step_block<float>(s, n, st);
    }
    int rc = launch_status();
    if (rc) return rc;
    for (int b = 0; b < s->B; ++b) s->h_pos_dec[b] += n;
    return RLT_OK;
}

// ---------------------------------------------------------------- graphs
// A transition block reads its positions from the device counters, so the
// kernels of kGraphBlocks consecutive blocks of n positions form one CUDA
// graph that serves every later stretch of the prefill: captured once per
// (state, n), then replayed.  Needs a stream other than the legacy default.
static constexpr int kGraphBlocks = 16;

static bool graphs_enabled(cudaStream_t st) {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("RLT_GRAPHS");
        v = (e && strcmp(e, "0") == 0) ? 0 : 1;
    }
    return v == 1 && st != nullptr && st != cudaStreamLegacy && st != cudaStreamPerThread;
}

// RLT_ROW_GROUPS=g: a captured run splits the rows into g contiguous groups
// whose chains of kernels run as concurrent branches of the graph (rows never
// interact; every kernel's result for a row is the same in any group).
// Read once.  Default, by the product rows R = B*n of a block: one group
// below 512, R/128 groups (at most 4) up to 1024 -- chains of 128-row
// products overlap each other's dependent-launch gaps -- and two beyond,
// where each product already fills the machine (measured: S5, 512 rows,
// 1.60M -> 1.72M tokens/s with four groups; the RLT-2 chunk workload, 4096
// product rows, best with two; the parity workload's 256 rows stay one
// chain).
static int row_groups(int B, int n) {
    static const int v = [] {
        const char* e = getenv("RLT_ROW_GROUPS");
        return e ? std::max(1, std::min(atoi(e), 8)) : 0;
    }();
    const long R = (long)B * n;
    const int g = v ? v : (R < 512 ? 1 : R <= 1024 ? (int)std::min<long>(4, R / 128) : 2);
    return std::max(1, std::min(g, B));
}

// RLT_GRAPH_CHAIN=1: inside a captured run, hand the state over and build the
// next merge input in one kernel (k_state_merge).  Off by default: measured
// against the two kernels the uncaptured blocks use, some rows came out
// different at the rounding level (cause not found), and the captured and
// uncaptured schedules must agree bit for bit.  Read once.
static bool graph_chain_enabled() {
    static const bool on = [] {
        const char* e = getenv("RLT_GRAPH_CHAIN");
        return e && strcmp(e, "1") == 0;
    }();
    return on;
}

static int run_graph(rlt_state* s, int n, cudaStream_t st) {
    const int span = kGraphBlocks * n;
    for (int b = 0; b < s->B; ++b) {
        if (s->h_pos_dec[b] + span > s->h_pos_enc[b]) return RLT_E_ORDER;
        if (s->h_pos_dec[b] + span > s->T_cap) return RLT_E_CAPACITY;
    }
    // profiling level 2 replays a twin graph whose attention launches are
    // bracketed by event nodes
    const bool timed = s->prof && s->prof_level >= 2;
    auto& gmap = timed ? s->graphs_prof : s->graphs;
    auto it = gmap.find(n);
    if (it == gmap.end()) {
        const bool prof = s->prof;
        s->prof = false;                  // no stream event records inside the capture
        s->prof_capture = timed;
        s->cap_recs.clear();
        const uint64_t l0 = rlt_kernel_launches();
        cudaGraph_t g = nullptr;
        cudaGraphExec_t ex = nullptr;
        // row groups: branches forked from and joined back into st (the
        // profiling twin issues them one after another on st, so that each
        // timed launch runs alone)
        int G = row_groups(s->B, n);
        while ((int)s->aux.size() < G - 1) {
            cudaStream_t a = nullptr;
            if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) {
                cudaGetLastError();
                break;
            }
            s->aux.push_back(a);
        }
        G = std::min(G, 1 + (int)s->aux.size());
        const bool branch = G > 1 && !timed;
        std::vector<cudaEvent_t> evs(branch ? G : 0, nullptr);
        bool ok = true;
        for (auto& ev : evs)
            ok = ok && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess;
        ok = ok && cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
        if (ok) {
            if (branch) {
                cudaEventRecord(evs[0], st);
                for (int k = 1; k < G; ++k) cudaStreamWaitEvent(s->aux[k - 1], evs[0], 0);
            }
            // consecutive one-position blocks hand the state to the next
            // block's merge input in one kernel
            const bool chain = n == 1 && s->m->cfg.variant != 0 && graph_chain_enabled();
            for (int gi = 0; gi < G; ++gi) {
                const int b0 = (int)((long)gi * s->B / G), b1 = (int)((long)(gi + 1) * s->B / G);
                cudaStream_t sg = branch && gi > 0 ? s->aux[gi - 1] : st;
                for (int k = 0; k < kGraphBlocks; ++k) {
                    s->prof_block = k;
                    const bool in = chain && k > 0, out = chain && k + 1 < kGraphBlocks;
                    if (s->m->cfg.dtype == RLT_DTYPE_BF16)
                        step_block<bf16>(s, n, sg, in, out, b0, b1 - b0);
                    else
                        step_block<float>(s, n, sg, in, out, b0, b1 - b0);
                }
            }
            if (branch)
                for (int k = 1; k < G; ++k) {
                    cudaEventRecord(evs[k], s->aux[k - 1]);
                    cudaStreamWaitEvent(st, evs[k], 0);
                }
            ok = cudaStreamEndCapture(st, &g) == cudaSuccess && g != nullptr;
        }
        for (auto& ev : evs)
            if (ev) cudaEventDestroy(ev);
        ok = ok && cudaGraphInstantiate(&ex, g, 0) == cudaSuccess;
        if (g) cudaGraphDestroy(g);
        const uint64_t captured = rlt_kernel_launches() - l0;
        g_launches.fetch_sub(captured);  // captured, not launched
        s->prof = prof;
        s->prof_capture = false;
        std::vector<rlt_state::CapRec> caps;
        caps.swap(s->cap_recs);
        if (!ok) {
            cudaGetLastError();
            if (ex) cudaGraphExecDestroy(ex);
            for (auto& c : caps) {
                cudaEventDestroy(c.a);
                cudaEventDestroy(c.b);
            }
            return RLT_E_UNSUPPORTED;     // the caller runs the blocks directly
        }
        it = gmap.emplace(n, rlt_state::Graph{ex, captured, std::move(caps)}).first;
    }
    double by = 0;
    if (s->prof) {
        std::vector<int32_t> saved = s->h_pos_dec;
        for (int k = 0; k < kGraphBlocks; ++k) {
            by += step_bytes(s, n);
            for (int b = 0; b < s->B; ++b) s->h_pos_dec[b] += n;
        }
        s->h_pos_dec = saved;
    }
    {
        ProfScope ps(s, RLT_PROF_STEP, st, by);
        if (cudaGraphLaunch(it->second.exec, st) != cudaSuccess) return RLT_E_DEVICE;
    }
    rlt_count_launch((int)it->second.launches);
    if (timed && !it->second.caps.empty()) {
        // the next replay re-records these events: read them now
        if (cudaStreamSynchronize(st) != cudaSuccess) return RLT_E_DEVICE;
        std::vector<int32_t> saved = s->h_pos_dec;
        for (auto& c : it->second.caps) {
            float t = 0.f;
            if (cudaEventElapsedTime(&t, c.a, c.b) != cudaSuccess) {
                cudaGetLastError();
                continue;
            }
            for (int b = 0; b < s->B; ++b) s->h_pos_dec[b] = saved[b] + c.block * n;
            const double cb = c.cls == RLT_PROF_XATTN ? xattn_bytes(s, n, c.b0, c.nb)
                              : c.cls == RLT_PROF_SWA ? swa_bytes(s, n, c.b0, c.nb) : 0.0;
            s->prof_recs.push_back({c.cls, nullptr, nullptr, cb, t, c.layer});
        }
        s->h_pos_dec = saved;
    }
    for (int b = 0; b < s->B; ++b) s->h_pos_dec[b] += span;
    return RLT_OK;
}

extern "C" int rlt_step(rlt_state* s, void* stream) {
    NvtxRange nvtx("rlt_step");
    if (!s) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    return run_block(s, 1, (cudaStream_t)stream);
}

extern "C" int rlt_prefill(rlt_state* s, int T, void* stream) {
    NvtxRange nvtx("rlt_prefill");
    if (!s || T < 0) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    const rlt_config& c = s->m->cfg;
    for (int b = 0; b < s->B; ++b) {
        if (s->h_pos_dec[b] + T > s->h_pos_enc[b]) return RLT_E_ORDER;
        if (s->h_pos_dec[b] + T > s->T_cap) return RLT_E_CAPACITY;
    }
    const cudaStream_t st = (cudaStream_t)stream;
    int done = 0;
    while (done < T) {
        const int pd = s->h_pos_dec[0];
        bool uniform = true;
        for (int b = 1; b < s->B; ++b) uniform &= s->h_pos_dec[b] == pd;
        int n = 1;
        if (uniform && c.variant == 2) n = std::min(T - done, c.chunk - pd % c.chunk);
        else if (uniform && c.variant == 0) n = std::min(T - done, s->n_dec_blk);
        // whole blocks of the regular shape go through a replayed graph
        const bool regular = c.variant == 1 || (c.variant == 2 && n == c.chunk) ||
                             (c.variant == 0 && n == s->n_dec_blk);
        if (regular && graphs_enabled(st) && T - done >= kGraphBlocks * n) {
            int rc = run_graph(s, n, st);
            if (rc == RLT_OK) {
                done += kGraphBlocks * n;
                continue;
            }
            if (rc != RLT_E_UNSUPPORTED) return rc;
        }
        int rc = run_block(s, n, st);
        if (rc) return rc;
        done += n;
    }
    return RLT_OK;
}

// ============================================================================
// readout
// ============================================================================
// logits fp32 [B][V] = W_out RMSNorm_out(s_t) of every row, into lbuf
static void readout_logits(rlt_state* s, float* lbuf, cudaStream_t st) {
    const rlt_model* m = s->m;
    const rlt_config& c = m->cfg;
    const int B = s->B, d = c.d, V = c.vocab;
    if (c.dtype == RLT_DTYPE_BF16) {
        rlt::launch_rmsnorm<bf16>(s->s, d, m->out_norm, (bf16*)s->Y, d, B, d, (float)c.eps, st);
        rlt::launch_gemm<bf16>((const bf16*)s->Y, d, (const bf16*)m->wout, d, lbuf, V, nullptr,
                               0, B, V, d, rlt::kStoreF32, st);
    } else {
        rlt::launch_rmsnorm<float>(s->s, d, m->out_norm, (float*)s->Y, d, B, d, (float)c.eps, st);
        rlt::launch_gemm<float>((const float*)s->Y, d, (const float*)m->wout, d, lbuf, V,
                                nullptr, 0, B, V, d, rlt::kStoreF32, st);
    }
}

extern "C" int rlt_readout(rlt_state* s, float* logits, int32_t* argmax, int32_t* sampled,
                           uint64_t seed, uint64_t step, float temperature, void* stream) {
    NvtxRange nvtx("rlt_readout");
    if (!s || !(temperature > 0.f)) return RLT_E_ARG;
    rlt_model* m = s->m;
    if (cudaSetDevice(m->device) != cudaSuccess) return RLT_E_DEVICE;
    const rlt_config& c = m->cfg;
    cudaStream_t st = (cudaStream_t)stream;
    const int B = s->B, V = c.vocab;
    const bool ld = logits && is_device_ptr(logits);
    const bool ad = argmax && is_device_ptr(argmax);
    const bool sd = sampled && is_device_ptr(sampled);
    float* lbuf = ld ? logits : s->logits;
    int32_t* abuf = argmax ? (ad ? argmax : s->ids) : nullptr;
    int32_t* sbuf = sampled ? (sd ? sampled : s->ids + B) : nullptr;
    readout_logits(s, lbuf, st);
    rlt::launch_sample(lbuf, V, B, abuf, sbuf, seed, step, temperature, st);
    int rc = launch_status();
    if (rc) return rc;
    if (logits && !ld &&
        cudaMemcpyAsync(logits, lbuf, (size_t)B * V * 4, cudaMemcpyDeviceToHost, st))
        return RLT_E_DEVICE;
    if (argmax && !ad &&
        cudaMemcpyAsync(argmax, abuf, (size_t)B * 4, cudaMemcpyDeviceToHost, st))
        return RLT_E_DEVICE;
    if (sampled && !sd &&
        cudaMemcpyAsync(sampled, sbuf, (size_t)B * 4, cudaMemcpyDeviceToHost, st))
        return RLT_E_DEVICE;
    // host outputs are valid on return (pinned memory would otherwise fill later)
    if (((logits && !ld) || (argmax && !ad) || (sampled && !sd)) &&
        cudaStreamSynchronize(st) != cudaSuccess)
        return RLT_E_DEVICE;
    return RLT_OK;
}

// [B][T_cap] fp32 and int32 buffers for the calls that stage per-position
// values or pieces of the caller's tokens, allocated on first use
static int call_scratch(rlt_state* s) {
    if (s->replay_lp) return RLT_OK;
    const size_t n = (size_t)s->B * s->T_cap * 4;
    int rc = salloc(s, (void**)&s->replay_lp, n);
    if (rc == RLT_OK) rc = salloc(s, (void**)&s->replay_tok, n);
    return rc;
}

// ============================================================================
// replay: log-probabilities of given tokens, each read before it is consumed
// ============================================================================
// The trainer's side of the replay contract: from the rows' current states
// (H_0 after a reset), append the tokens to the encoder in one parallel pass
// (causal, so later tokens do not change earlier features), then per position
// read log p(token | everything before it) from the current s and consume the
// token with one transition (jiphyeonjeon review §6.2, eq. 5.3-5.5;
// greeksharifa App. D.3, F.4).
extern "C" int rlt_replay_logprobs(rlt_state* s, const int32_t* tokens, int n, float* logprobs,
                                   float temperature, void* stream) {
    NvtxRange nvtx("rlt_replay_logprobs");
    if (!s || !tokens || !logprobs || n < 0 || !(temperature > 0.f)) return RLT_E_ARG;
    if (n == 0) return RLT_OK;
    for (int b = 0; b < s->B; ++b)
        if (s->h_pos_dec[b] != s->h_pos_enc[b]) return RLT_E_ORDER;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    const cudaStream_t st = (cudaStream_t)stream;
    const int B = s->B, V = s->m->cfg.vocab;
    if (int rc = call_scratch(s)) return rc;
    const bool tdev = is_device_ptr(tokens), odev = is_device_ptr(logprobs);
    // capacity and (host) token range are checked here, before anything runs
    int rc = rlt_encode(s, tokens, n, stream);
    if (rc) return rc;
    const int32_t* ids = tokens;
    if (!tdev) {
        if (cudaMemcpyAsync(s->replay_tok, tokens, (size_t)B * n * 4, cudaMemcpyHostToDevice,
                            st) != cudaSuccess)
            return RLT_E_DEVICE;
        ids = s->replay_tok;
    }
    float* out = odev ? logprobs : s->replay_lp;
    for (int j = 0; j < n; ++j) {
        readout_logits(s, s->logits, st);
        rlt::launch_logprob(s->logits, V, B, ids + j, n, out + j, n, temperature, s->err, st);
        rc = launch_status();
        if (rc) return rc;
        rc = run_block(s, 1, st);
        if (rc) return rc;
    }
    if (!odev) {
        if (cudaMemcpyAsync(logprobs, out, (size_t)B * n * 4, cudaMemcpyDeviceToHost, st) !=
                cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess)
            return RLT_E_DEVICE;
    }
    return RLT_OK;
}

// ============================================================================
// packed documents: a row restarts from H_0 where a document starts
// ============================================================================
// Independent documents packed one after another in a row reset the
// recurrent output, the window rings, the encoder cache and the positions at
// each document start, so no state and no attention crosses the boundary
// (jiphyeonjeon review §6.1; greeksharifa App. F).  The columns are cut
// wherever any row starts a document; each piece is encoded and consumed by
// every row, after the rows that start a document at the piece's first column
// are reset.  Rows then sit at different positions, which every kernel
// handles through its row's own counters.
extern "C" int rlt_prefill_packed(rlt_state* s, const int32_t* tokens, const uint8_t* doc_start,
                                  int n, void* stream) {
    NvtxRange nvtx("rlt_prefill_packed");
    if (!s || !tokens || !doc_start || n < 0) return RLT_E_ARG;
    if (n == 0) return RLT_OK;
    const int B = s->B;
    for (int b = 0; b < B; ++b)
        if (s->h_pos_dec[b] != s->h_pos_enc[b]) return RLT_E_ORDER;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    if (is_device_ptr(doc_start)) return RLT_E_ARG;     // read on the host below
    const bool tdev = is_device_ptr(tokens);
    // everything that could fail part-way is checked before the first piece
    for (int b = 0; b < B; ++b) {
        int p = s->h_pos_enc[b];
        for (int j = 0; j < n; ++j) {
            p = doc_start[(size_t)b * n + j] ? 1 : p + 1;
            if (p > s->T_cap) return RLT_E_CAPACITY;
            if (!tdev && (tokens[(size_t)b * n + j] < 0 ||
                          tokens[(size_t)b * n + j] >= s->m->cfg.vocab))
                return RLT_E_ARG;
        }
    }
    if (tdev)
        if (int rc = call_scratch(s)) return rc;
    const cudaStream_t st = (cudaStream_t)stream;
    auto starts_at = [&](int j) {
        for (int b = 0; b < B; ++b)
            if (doc_start[(size_t)b * n + j]) return true;
        return false;
    };
    std::vector<int32_t> piece_h, rows;
    for (int j0 = 0; j0 < n;) {
        int j1 = j0 + 1;
        while (j1 < n && !starts_at(j1)) ++j1;
        const int len = j1 - j0;
        rows.clear();
        for (int b = 0; b < B; ++b)
            if (doc_start[(size_t)b * n + j0]) rows.push_back(b);
        if (!rows.empty())
            if (int rc = rlt_state_reset(s, rows.data(), (int)rows.size(), stream)) return rc;
        const int32_t* piece;
        if (tdev) {
            if (cudaMemcpy2DAsync(s->replay_tok, (size_t)len * 4, tokens + j0, (size_t)n * 4,
                                  (size_t)len * 4, B, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
                return RLT_E_DEVICE;
            piece = s->replay_tok;
        } else {
            // rlt_encode stages a pageable host piece before it returns
            piece_h.resize((size_t)B * len);
            for (int b = 0; b < B; ++b)
                memcpy(&piece_h[(size_t)b * len], tokens + (size_t)b * n + j0, (size_t)len * 4);
            piece = piece_h.data();
        }
        if (int rc = rlt_encode(s, piece, len, stream)) return rc;
        if (int rc = rlt_prefill(s, len, stream)) return rc;
        j0 = j1;
    }
    return RLT_OK;
}

// ============================================================================
// reset, positions, export, errors
// ============================================================================
extern "C" int rlt_state_reset(rlt_state* s, const int32_t* rows, int n, void* stream) {
    NvtxRange nvtx("rlt_state_reset");
    if (!s) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    cudaStream_t st = (cudaStream_t)stream;
    if (!rows) {
        rlt::launch_reset_rows(nullptr, s->B, s->m->s_star, s->s, s->Rr, s->pos_enc, s->pos_dec,
                               s->m->cfg.d, st);
        std::fill(s->h_pos_enc.begin(), s->h_pos_enc.end(), 0);
        std::fill(s->h_pos_dec.begin(), s->h_pos_dec.end(), 0);
        return launch_status();
    }
    if (n < 0 || n > s->B) return RLT_E_ARG;
    for (int i = 0; i < n; ++i)
        if (rows[i] < 0 || rows[i] >= s->B) return RLT_E_ARG;
    if (n == 0) return RLT_OK;
    if (cudaMemcpyAsync(s->rows, rows, (size_t)n * 4, cudaMemcpyHostToDevice, st))
        return RLT_E_DEVICE;
    rlt::launch_reset_rows(s->rows, n, s->m->s_star, s->s, s->Rr, s->pos_enc, s->pos_dec,
                           s->m->cfg.d, st);
    // the host copy of `rows` may be reused by the caller once the copy is done
    if (cudaStreamSynchronize(st) != cudaSuccess) return RLT_E_DEVICE;
    for (int i = 0; i < n; ++i) s->h_pos_enc[rows[i]] = s->h_pos_dec[rows[i]] = 0;
    return launch_status();
}

extern "C" int rlt_state_positions(const rlt_state* s, int32_t* pos_enc, int32_t* pos_dec) {
    if (!s) return RLT_E_ARG;
    if (pos_enc) memcpy(pos_enc, s->h_pos_enc.data(), (size_t)s->B * 4);
    if (pos_dec) memcpy(pos_dec, s->h_pos_dec.data(), (size_t)s->B * 4);
    return RLT_OK;
}

extern "C" int rlt_state_read(rlt_state* s, int part, void* dst, size_t nbytes,
                              size_t* nbytes_out, void* stream) {
    if (!s) return RLT_E_ARG;
    const void* src = nullptr;
    size_t sz = 0;
    const size_t B = s->B, d = s->m->cfg.d, elt = s->m->elt;
    switch (part) {
        case RLT_PART_S: src = s->s; sz = B * d * 4; break;
        case RLT_PART_R: src = s->Rr; sz = B * d * 4; break;
        case RLT_PART_E: src = s->e; sz = B * s->T_cap * d * 4; break;
        case RLT_PART_MEM: src = s->mem; sz = B * s->mem_row * elt; break;
        case RLT_PART_RING: src = s->ring; sz = B * s->ring_row * elt; break;
        case RLT_PART_ENC: src = s->enc; sz = B * s->enc_row * elt; break;
        default: return RLT_E_ARG;
    }
    if (nbytes_out) *nbytes_out = sz;
    if (!dst) return RLT_OK;
    if (nbytes != sz) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    cudaStream_t st = (cudaStream_t)stream;
    const bool dev = is_device_ptr(dst);
    if (cudaMemcpyAsync(dst, src, sz, dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost,
                        st))
        return RLT_E_DEVICE;
    if (!dev && cudaStreamSynchronize(st)) return RLT_E_DEVICE;
    return RLT_OK;
}

// ============================================================================
// exact prefix snapshots of one row
// ============================================================================
// A row resumes exactly from: the encoder cache C^E and the memory M of every
// encoded position, the decoder state s (and the RLT-2 register R), the window
// rings C^D, the encoder outputs e_t that transitions still have to merge,
// both positions, and the identity of the weights and config the row was
// built under (jiphyeonjeon review §6.5, multi-turn serving; greeksharifa
// App. E, App. H).  The byte layout is the one include/rlt.h documents; it
// does not depend on the state's batch or max_len.
namespace {
constexpr size_t kSnapHeader = RLT_SNAPSHOT_HEADER_BYTES;
constexpr uint32_t kSnapVersion = 1;

struct SnapGeom {
    size_t d, dh, elt;
    size_t enc_planes, mem_planes;   // [T_cap][d_h] planes of one row's C^E and M
    size_t ring;                     // elements of one row's window rings
};

SnapGeom snap_geom(const rlt_config& c) {
    SnapGeom g;
    g.d = (size_t)c.d;
    g.dh = (size_t)(c.d / c.heads);
    g.elt = c.dtype == RLT_DTYPE_BF16 ? 2 : 4;
    g.enc_planes = (size_t)c.n_enc * 2 * c.heads;
    g.mem_planes = (size_t)(c.n_dec > 0 ? c.groups : 0) * 2 * c.heads;
    g.ring = (size_t)c.n_dec * 2 * c.heads * (size_t)std::max(0, c.window - 1) * g.dh;
    return g;
}

size_t snap_bytes(const SnapGeom& g, int pos_enc) {
    const size_t p = (size_t)pos_enc;
    return kSnapHeader + 2 * g.d * 4 + p * g.d * 4 +
           (g.enc_planes + g.mem_planes) * p * g.dh * g.elt + g.ring * g.elt;
}

void snap_write_header(uint8_t* h, const rlt_config& c, uint64_t checksum, int32_t pos_enc,
                       int32_t pos_dec) {
    memset(h, 0, kSnapHeader);
    memcpy(h, "RLTS", 4);
    memcpy(h + 4, &kSnapVersion, 4);
    memcpy(h + 8, &checksum, 8);
    memcpy(h + 16, &pos_enc, 4);
    memcpy(h + 20, &pos_dec, 4);
    const int32_t f[12] = {c.vocab, c.d,     c.heads, c.n_enc,   c.n_dec, c.ffn,
                           c.window, c.groups, c.chunk, c.variant, c.tied,  c.dtype};
    memcpy(h + 24, f, sizeof f);
    memcpy(h + 72, &c.alpha, 8);
    memcpy(h + 80, &c.eps, 8);
    memcpy(h + 88, &c.rope_base, 8);
}

// Reads and checks a header against the snapshot's total size.  The bounds
// keep every size product below 2^63.
int snap_read_header(const uint8_t* h, size_t nbytes, rlt_config* c, uint64_t* checksum,
                     int32_t* pos_enc, int32_t* pos_dec) {
    if (nbytes < kSnapHeader || memcmp(h, "RLTS", 4) != 0) return RLT_E_SNAPSHOT;
    uint32_t ver;
    memcpy(&ver, h + 4, 4);
    if (ver != kSnapVersion) return RLT_E_SNAPSHOT;
    for (size_t i = 96; i < kSnapHeader; ++i)
        if (h[i]) return RLT_E_SNAPSHOT;
    memcpy(checksum, h + 8, 8);
    memcpy(pos_enc, h + 16, 4);
    memcpy(pos_dec, h + 20, 4);
    int32_t f[12];
    memcpy(f, h + 24, sizeof f);
    c->vocab = f[0]; c->d = f[1]; c->heads = f[2]; c->n_enc = f[3]; c->n_dec = f[4];
    c->ffn = f[5]; c->window = f[6]; c->groups = f[7]; c->chunk = f[8]; c->variant = f[9];
    c->tied = f[10]; c->dtype = f[11];
    memcpy(&c->alpha, h + 72, 8);
    memcpy(&c->eps, h + 80, 8);
    memcpy(&c->rope_base, h + 88, 8);
    if (c->d <= 0 || c->d > (1 << 16) || c->heads <= 0 || c->d % c->heads || c->n_enc < 0 ||
        c->n_enc > 1024 || c->n_dec < 0 || c->n_dec > 1024 || c->window < 1 ||
        c->window > (1 << 24) || c->groups < 1 || c->groups > 1024 ||
        (c->dtype != RLT_DTYPE_F32 && c->dtype != RLT_DTYPE_BF16))
        return RLT_E_SNAPSHOT;
    if (*pos_enc < 0 || *pos_enc > (1 << 28) || *pos_dec < 0 || *pos_dec > *pos_enc)
        return RLT_E_SNAPSHOT;
    if (nbytes != snap_bytes(snap_geom(*c), *pos_enc)) return RLT_E_SNAPSHOT;
    return RLT_OK;
}

bool same_config(const rlt_config& a, const rlt_config& b) {
    return a.vocab == b.vocab && a.d == b.d && a.heads == b.heads && a.n_enc == b.n_enc &&
           a.n_dec == b.n_dec && a.ffn == b.ffn && a.window == b.window &&
           a.groups == b.groups && a.chunk == b.chunk && a.variant == b.variant &&
           a.tied == b.tied && a.dtype == b.dtype && memcmp(&a.alpha, &b.alpha, 8) == 0 &&
           memcmp(&a.eps, &b.eps, 8) == 0 && memcmp(&a.rope_base, &b.rope_base, 8) == 0;
}

// Copies between one row of a state and a packed snapshot: the snapshot's
// sections in their order, each section a plain copy except C^E and M, whose
// first pos_enc positions of every [T_cap][d_h] plane are packed.
struct SnapCopier {
    rlt_state* s;
    int row, pos;
    SnapGeom g;
    uint8_t* snap;
    bool to_snap;                // state -> snapshot (save) or back (load)
    cudaMemcpyKind kind;
    cudaStream_t st;
    size_t off = kSnapHeader;
    cudaError_t e = cudaSuccess;

    void flat(void* state_part, size_t bytes) {
        if (e == cudaSuccess && bytes)
            e = to_snap ? cudaMemcpyAsync(snap + off, state_part, bytes, kind, st)
                        : cudaMemcpyAsync(state_part, snap + off, bytes, kind, st);
        off += bytes;
    }
    void planes(void* state_row, size_t n_planes) {
        const size_t w = (size_t)pos * g.dh * g.elt, pitch = (size_t)s->T_cap * g.dh * g.elt;
        if (e == cudaSuccess && w && n_planes)
            e = to_snap ? cudaMemcpy2DAsync(snap + off, w, state_row, pitch, w, n_planes, kind, st)
                        : cudaMemcpy2DAsync(state_row, pitch, snap + off, w, w, n_planes, kind, st);
        off += w * n_planes;
    }
    void all() {
        const size_t r = (size_t)row;
        flat(s->s + r * g.d, g.d * 4);
        flat(s->Rr + r * g.d, g.d * 4);
        flat(s->e + r * s->T_cap * g.d, (size_t)pos * g.d * 4);
        planes((uint8_t*)s->enc + r * s->enc_row * g.elt, g.enc_planes);
        planes((uint8_t*)s->mem + r * s->mem_row * g.elt, g.mem_planes);
        flat((uint8_t*)s->ring + r * s->ring_row * g.elt, g.ring * g.elt);
    }
};
}  // namespace

extern "C" int rlt_snapshot_info(const void* snap, size_t nbytes, rlt_config* cfg,
                                 int32_t* pos_enc, int32_t* pos_dec) {
    if (!snap) return RLT_E_ARG;
    rlt_config c;
    uint64_t ck;
    int32_t pe, pd;
    const int rc = snap_read_header((const uint8_t*)snap, nbytes, &c, &ck, &pe, &pd);
    if (rc) return rc;
    if (cfg) *cfg = c;
    if (pos_enc) *pos_enc = pe;
    if (pos_dec) *pos_dec = pd;
    return RLT_OK;
}

extern "C" int rlt_state_save(rlt_state* s, int row, void* dst, size_t nbytes,
                              size_t* nbytes_out, void* stream) {
    NvtxRange nvtx("rlt_state_save");
    if (!s || row < 0 || row >= s->B) return RLT_E_ARG;
    const rlt_model* m = s->m;
    const SnapGeom g = snap_geom(m->cfg);
    const int32_t pe = s->h_pos_enc[row], pd = s->h_pos_dec[row];
    const size_t sz = snap_bytes(g, pe);
    if (nbytes_out) *nbytes_out = sz;
    if (!dst) return RLT_OK;
    if (nbytes != sz) return RLT_E_ARG;
    if (cudaSetDevice(m->device) != cudaSuccess) return RLT_E_DEVICE;
    const cudaStream_t st = (cudaStream_t)stream;
    const bool dev = is_device_ptr(dst);
    uint8_t hdr[kSnapHeader];
    snap_write_header(hdr, m->cfg, m->checksum, pe, pd);
    SnapCopier cp{s, row, pe, g, (uint8_t*)dst, true,
                  dev ? cudaMemcpyDeviceToDevice : cudaMemcpyDeviceToHost, st};
    if (dev) cp.e = cudaMemcpyAsync(dst, hdr, kSnapHeader, cudaMemcpyHostToDevice, st);
    else memcpy(dst, hdr, kSnapHeader);
    cp.all();
    // the header's host copy and a host destination are done with on return
    if (cp.e == cudaSuccess) cp.e = cudaStreamSynchronize(st);
    if (cp.e != cudaSuccess || cp.off != sz) {
        cudaGetLastError();
        return RLT_E_DEVICE;
    }
    return RLT_OK;
}

extern "C" int rlt_state_load(rlt_state* s, int row, const void* src, size_t nbytes,
                              void* stream) {
    NvtxRange nvtx("rlt_state_load");
    if (!s || !src || row < 0 || row >= s->B) return RLT_E_ARG;
    const rlt_model* m = s->m;
    if (cudaSetDevice(m->device) != cudaSuccess) return RLT_E_DEVICE;
    const cudaStream_t st = (cudaStream_t)stream;
    const bool dev = is_device_ptr(src);
    uint8_t hdr[kSnapHeader];
    if (nbytes < kSnapHeader) return RLT_E_SNAPSHOT;
    if (dev) {
        if (cudaMemcpyAsync(hdr, src, kSnapHeader, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
            cudaStreamSynchronize(st) != cudaSuccess) {
            cudaGetLastError();
            return RLT_E_DEVICE;
        }
    } else {
        memcpy(hdr, src, kSnapHeader);
    }
    rlt_config c;
    uint64_t ck;
    int32_t pe, pd;
    int rc = snap_read_header(hdr, nbytes, &c, &ck, &pe, &pd);
    if (rc) return rc;
    if (ck != m->checksum || !same_config(c, m->cfg)) return RLT_E_SNAPSHOT;
    if (pe > s->T_cap) return RLT_E_CAPACITY;
    const SnapGeom g = snap_geom(m->cfg);
    SnapCopier cp{s, row, pe, g, (uint8_t*)const_cast<void*>(src), false,
                  dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, st};
    cp.all();
    // positions straight from the snapshot's header fields
    const uint8_t* sp = (const uint8_t*)src;
    if (cp.e == cudaSuccess) cp.e = cudaMemcpyAsync(s->pos_enc + row, sp + 16, 4, cp.kind, st);
    if (cp.e == cudaSuccess) cp.e = cudaMemcpyAsync(s->pos_dec + row, sp + 20, 4, cp.kind, st);
    // a host source may be freed on return
    if (cp.e == cudaSuccess) cp.e = cudaStreamSynchronize(st);
    if (cp.e != cudaSuccess || cp.off != nbytes) {
        cudaGetLastError();
        return RLT_E_DEVICE;
    }
    s->h_pos_enc[row] = pe;
    s->h_pos_dec[row] = pd;
    return RLT_OK;
}

extern "C" int rlt_selftest_wait(rlt_state* s, int kind, uint32_t polls, void* stream) {
    NvtxRange nvtx("rlt_selftest_wait");
    if (!s || (kind != 0 && kind != 1) || polls == 0 || polls > (1u << 24)) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    rlt::launch_selftest_wait(kind, polls, s->err, (cudaStream_t)stream);
    return launch_status();
}

extern "C" uint32_t rlt_build_flags(void) { return RLT_DEBUG ? RLT_BUILD_DEBUG : 0u; }

extern "C" int rlt_debug_set_positions(rlt_state* s, int row, int32_t pos_enc, int32_t pos_dec,
                                       void* stream) {
    if (!RLT_DEBUG) return RLT_E_UNSUPPORTED;
    if (!s || row < 0 || row >= s->B) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    const cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(s->pos_enc + row, &pos_enc, 4, cudaMemcpyHostToDevice, st) ||
        cudaMemcpyAsync(s->pos_dec + row, &pos_dec, 4, cudaMemcpyHostToDevice, st) ||
        cudaStreamSynchronize(st))
        return RLT_E_DEVICE;
    return RLT_OK;
}

extern "C" int rlt_state_check(rlt_state* s, void* stream) {
    if (!s) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RLT_E_DEVICE;
    int w = 0;
    if (cudaMemcpy(&w, s->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return RLT_E_DEVICE;
    if (w != 0 && cudaMemset(s->err, 0, 4) != cudaSuccess) return RLT_E_DEVICE;
    const int g = rlt::read_and_clear_device_error();
    const int ga = rlt::read_and_clear_attn_error();
    const int gp = rlt::read_and_clear_persist_error();
    const int gm = rlt::read_and_clear_mq_error();
    const int gs = rlt::read_and_clear_sq_error();
    if (g < 0 || ga < 0 || gp < 0 || gm < 0 || gs < 0) return RLT_E_DEVICE;
    if (w == 0) w = g ? g : (ga ? ga : (gp ? gp : (gm ? gm : gs)));
    if (w == rlt::kDevTimeout) return RLT_E_TIMEOUT;
    if (w == rlt::kDevBounds) return RLT_E_ARG;
    if (w == rlt::kDevOrder) return RLT_E_ORDER;
    if (w == rlt::kDevCapacity) return RLT_E_CAPACITY;
    return w ? RLT_E_DEVICE : RLT_OK;
}

extern "C" uint64_t rlt_kernel_launches(void) { return g_launches.load(); }

extern "C" int rlt_profile_enable(rlt_state* s, int on) {
    if (!s) return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    if (cudaDeviceSynchronize() != cudaSuccess) return RLT_E_DEVICE;
    for (auto& r : s->prof_recs) {
        if (r.a) s->prof_pool.push_back(r.a);
        if (r.b) s->prof_pool.push_back(r.b);
    }
    s->prof_recs.clear();
    s->prof = on != 0;
    s->prof_level = on < 0 ? 0 : on;
    return RLT_OK;
}

extern "C" int rlt_profile_query(rlt_state* s, int cls, uint64_t* launches, double* total_ms,
                                 double* bytes, void* stream) {
    // cls + RLT_PROF_NCLS * (l + 1): the class's launches in decoder layer l only
    if (!s || cls < 0 || cls >= RLT_PROF_NCLS * (1 + std::max(0, s->m->cfg.n_dec)))
        return RLT_E_ARG;
    if (cudaSetDevice(s->m->device) != cudaSuccess) return RLT_E_DEVICE;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return RLT_E_DEVICE;
    const int base = cls % RLT_PROF_NCLS, want_layer = cls / RLT_PROF_NCLS - 1;
    uint64_t n = 0;
    double ms = 0, by = 0;
    for (auto& r : s->prof_recs) {
        if (r.cls != base || (want_layer >= 0 && r.layer != want_layer)) continue;
        float t = r.ms;
        if (!r.a) {                      // resolved right after its graph replay
            ++n;
            ms += t;
            by += r.bytes;
            continue;
        }
        if (cudaEventSynchronize(r.b) != cudaSuccess ||
            cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            return RLT_E_DEVICE;
        ++n;
        ms += t;
        by += r.bytes;
    }
    if (launches) *launches = n;
    if (total_ms) *total_ms = ms;
    if (bytes) *bytes = by;
    return RLT_OK;
}

extern "C" const char* rlt_strerror(int code) {
    switch (code) {
        case RLT_OK: return "ok";
        case RLT_E_ARG: return "invalid argument";
        case RLT_E_OOM: return "out of memory";
        case RLT_E_CAPACITY: return "position would exceed the state's max_len";
        case RLT_E_ORDER: return "transition without an encoded token at that position";
        case RLT_E_BLOB: return "bad weight blob (magic, version, manifest or checksum)";
        case RLT_E_DEVICE: return "CUDA error";
        case RLT_E_TIMEOUT: return "bounded device wait gave up";
        case RLT_E_UNSUPPORTED: return "unsupported configuration";
        case RLT_E_SNAPSHOT: return "bad snapshot (magic, version, size) or taken under other weights";
        default: return "unknown error";
    }
}

// ============================================================================
// readout of caller-supplied state vectors, without allocating
// ============================================================================
// rlt_readout keeps its scratch (normalised rows, logits, ids) in the state.
// A caller that holds only a model -- scoring state vectors it exported with
// rlt_state_read, or candidates of its own -- has no state to lend, and some
// such callers must not allocate at all: a serving process whose memory pool
// already owns the rest of the device (a cudaMalloc there fails or evicts),
// or one whose other streams are in flight (cudaMalloc / cudaFree may
// synchronise the device and stall them).  This entry point therefore keeps
// its scratch in a file-scope device array, sized once at build time, and
// runs the same three kernels as rlt_readout on it.
namespace {
static __device__ __align__(256) unsigned char g_rows_scratch[RLT_READOUT_ROWS_SCRATCH_BYTES];
constexpr int kScratchDevices = 64;
void* g_rows_scratch_at[kScratchDevices];    // device address, looked up once per device
std::mutex g_rows_scratch_mu;

void* rows_scratch(int device) {
    std::lock_guard<std::mutex> lk(g_rows_scratch_mu);
    if (!g_rows_scratch_at[device]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_rows_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_rows_scratch_at[device] = p;
    }
    return g_rows_scratch_at[device];
}
}  // namespace

extern "C" int rlt_readout_rows(const rlt_model* m, const float* s_rows, int rows, float* logits,
                                int32_t* argmax, int32_t* sampled, uint64_t seed, uint64_t step,
                                float temperature, void* stream) {
    NvtxRange nvtx("rlt_readout_rows");
    if (!m || !s_rows || rows < 0 || !(temperature > 0.f)) return RLT_E_ARG;
    if (m->device < 0 || m->device >= kScratchDevices) return RLT_E_DEVICE;
    if (cudaSetDevice(m->device) != cudaSuccess) return RLT_E_DEVICE;
    if (rows == 0) return RLT_OK;
    if (!is_device_ptr(s_rows)) return RLT_E_ARG;
    const rlt_config& c = m->cfg;
    const int d = c.d, V = c.vocab;
    const bool bf = c.dtype == RLT_DTYPE_BF16;
    const bool ld = logits && is_device_ptr(logits);
    const bool ad = argmax && is_device_ptr(argmax);
    const bool sd = sampled && is_device_ptr(sampled);
    // scratch: [normalised rows, storage type][logits fp32, unless the
    // caller's are on the device][argmax, sampled int32], each 256-aligned;
    // every byte read is written earlier in the same call
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t off_l = up((size_t)rows * d * (bf ? 2 : 4));
    const size_t off_i = off_l + (ld ? 0 : up((size_t)rows * V * 4));
    const size_t need = off_i + up((size_t)rows * 2 * 4);
    if (need > (size_t)RLT_READOUT_ROWS_SCRATCH_BYTES) return RLT_E_ARG;
    unsigned char* base = (unsigned char*)rows_scratch(m->device);
    if (!base) return RLT_E_DEVICE;
    cudaStream_t st = (cudaStream_t)stream;
    float* lbuf = ld ? logits : (float*)(base + off_l);
    int32_t* ids = (int32_t*)(base + off_i);
    int32_t* abuf = argmax ? (ad ? argmax : ids) : nullptr;
    int32_t* sbuf = sampled ? (sd ? sampled : ids + rows) : nullptr;
    if (bf) {
        bf16* Y = (bf16*)base;
        rlt::launch_rmsnorm<bf16>(s_rows, d, m->out_norm, Y, d, rows, d, (float)c.eps, st);
        rlt::launch_gemm<bf16>(Y, d, (const bf16*)m->wout, d, lbuf, V, nullptr, 0, rows, V, d,
                               rlt::kStoreF32, st);
    } else {
        float* Y = (float*)base;
        rlt::launch_rmsnorm<float>(s_rows, d, m->out_norm, Y, d, rows, d, (float)c.eps, st);
        rlt::launch_gemm<float>(Y, d, (const float*)m->wout, d, lbuf, V, nullptr, 0, rows, V, d,
                                rlt::kStoreF32, st);
    }
    rlt::launch_sample(lbuf, V, rows, abuf, sbuf, seed, step, temperature, st);
    int rc = launch_status();
    if (rc) return rc;
    if (logits && !ld &&
        cudaMemcpyAsync(logits, lbuf, (size_t)rows * V * 4, cudaMemcpyDeviceToHost, st))
        return RLT_E_DEVICE;
    if (argmax && !ad &&
        cudaMemcpyAsync(argmax, abuf, (size_t)rows * 4, cudaMemcpyDeviceToHost, st))
        return RLT_E_DEVICE;
    if (sampled && !sd &&
        cudaMemcpyAsync(sampled, sbuf, (size_t)rows * 4, cudaMemcpyDeviceToHost, st))
        return RLT_E_DEVICE;
    // host outputs are valid on return, and the copies out of the shared
    // array have finished before the next call can overwrite it
    if (((logits && !ld) || (argmax && !ad) || (sampled && !sd)) &&
        cudaStreamSynchronize(st) != cudaSuccess)
        return RLT_E_DEVICE;
    return RLT_OK;
}
