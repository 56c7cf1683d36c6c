/*
 * rlt.h -- C ABI of the RLT transition engine (librlt.so, sm_100a).
 *
 * The Recurrent Looped Transformer carries a full decoder state
 * H_t = (s_t, C^D_t) -- the last decoder output and one sliding-window
 * key/value cache per decoder layer -- across every token, prompt and
 * response alike, and reads a prefix-restricted memory built by a causal
 * encoder (jiphyeonjeon.kr review "Recurrent Looped Transformer", §2-§3;
 * greeksharifa.github.io "Recurrent Looped Transformer 요약 설명", §2.1-§2.7).
 * This library runs that transition for a batch of independent sequences
 * ("rows") on one GPU.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Return value: RLT_OK (0) on success, a negative RLT_E_* code otherwise.
 *   Nothing traps; device-side failures (a bounded wait that gave up) set a
 *   sticky per-state error word that rlt_state_check() reports.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Calls are stream-ordered and asynchronous unless stated.
 * - Ownership: models and states are library-owned and freed by their
 *   destroy call.  Caller buffers (tokens, logits, ids) stay caller-owned; the
 *   library never frees or retains them past the call's stream work.
 * - Host or device pointers: every caller buffer may be host memory (pageable
 *   or pinned) or device memory of the state's device; the library checks with
 *   cudaPointerGetAttributes and stages host buffers through its own device
 *   copies on `stream`.  Host outputs are valid after `stream` synchronises.
 * - Rows are independent: row r's results do not depend on the batch size or
 *   on other rows' tokens, bit for bit (greeksharifa App. C.1, batching
 *   independent sequences).
 * - Positions are 1-based; BOS is position 1 (greeksharifa App. I).
 * - Threads: one model or state must not be used by two host threads at
 *   once; different states may run on different threads and streams.  A
 *   bounded wait that gives up inside the GEMMs or the bulk-copy attention
 *   kernels records it in a device-wide word (other kernels use the state's
 *   own), which the first rlt_state_check on that device to run afterwards
 *   reports and clears.
 */
#ifndef RLT_H
#define RLT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RLT_OK             0
#define RLT_E_ARG         -1  /* bad argument (null pointer, size, row index)            */
#define RLT_E_OOM         -2  /* device or host allocation failed                         */
#define RLT_E_CAPACITY    -3  /* a row's position would exceed the state's max_len        */
#define RLT_E_ORDER       -4  /* transition without an encoded token (pos_dec >= pos_enc) */
#define RLT_E_BLOB        -5  /* weight blob: bad magic, version, manifest or checksum    */
#define RLT_E_DEVICE      -6  /* a CUDA call failed (no device, launch error, fault)      */
#define RLT_E_TIMEOUT     -7  /* a bounded device wait gave up                            */
#define RLT_E_UNSUPPORTED -8  /* configuration this build does not run                    */
#define RLT_E_SNAPSHOT    -9  /* snapshot: bad magic, version or size, or other weights   */

#define RLT_DTYPE_F32  0
#define RLT_DTYPE_BF16 1

typedef struct rlt_model rlt_model;  /* weights on one device + config              */
typedef struct rlt_state rlt_state;  /* s, R, C^D rings, C^E, memory, e, positions   */

/* Model hyper-parameters as stored in the blob header. */
typedef struct rlt_config {
    int32_t vocab, d, heads, n_enc, n_dec, ffn, window, groups, chunk, variant, tied, dtype;
    double alpha, eps, rope_base;
} rlt_config;

/* Load a weight blob (host memory, copied; the caller may free it on return)
 * onto `device`.  Blob = 256-byte header (magic "RLTB", version 1, the
 * rlt_config fields, seed, tensor count, payload size, checksum) followed by
 * named tensor records in the fixed manifest order of the config.  Errors:
 * RLT_E_BLOB (bad magic/version/manifest/checksum), RLT_E_UNSUPPORTED (head
 * size other than 16, 32, 64, 128, or width d above 2048), RLT_E_DEVICE,
 * RLT_E_OOM.  Models on several devices may share a process: every call
 * makes its model's device current, and kernel attributes are set per
 * device. */
int rlt_create(const void* blob, size_t nbytes, int device, rlt_model** out);
void rlt_destroy(rlt_model* model);
int rlt_model_config(const rlt_model* model, rlt_config* out);

/* Allocate the per-row state for `batch` rows of up to `max_len` positions:
 * encoder cache C^E [L_E][2][h][max_len][d_h], memory M [G][2][h][max_len][d_h],
 * window rings C^D [L_D][2][h][W-1][d_h] (all in the model dtype), e_t
 * [max_len][d] fp32, s and R [d] fp32 -- the storage bound of the paper's
 * eq. 3.3 (jiphyeonjeon review §4.2) -- plus scratch for one call.  The
 * state starts reset (H_0).  Library-owned.  RLT_E_ARG for batch or max_len
 * <= 0; RLT_E_OOM when an allocation fails, or before allocating when
 * batch x (max_len + W + B_c + 16) x (3d + 2f' + vocab) x 4 x (2(L_E + L_D + G)
 * + 8), f' = f rounded up to 64 -- a bound on every buffer's bytes -- exceeds
 * 2^60. */
int rlt_state_create(rlt_model* model, int batch, int max_len, rlt_state** out);
void rlt_state_destroy(rlt_state* state);

/* Bytes of the per-row state proper (eq. 3.3 terms) and of everything the
 * state allocated on the device (state + scratch). */
int rlt_state_bytes(const rlt_state* state, size_t* per_row_state, size_t* total_device);

/* H_0 = (s_star, empty) for `n` rows listed in host array `rows` (NULL = all
 * rows): s = R = s_star, caches emptied, positions 0 (jiphyeonjeon review §3.1;
 * per-document reset, §6.1). */
int rlt_state_reset(rlt_state* state, const int32_t* rows, int n, void* stream);

/* Encode `n` tokens per row (tokens: int32 [batch][n], host or device) at
 * positions pos_enc+1..pos_enc+n: appends e_t, C^E and the memory entries
 * k^g_t = RoPE_t(W^g_K RMSNorm_E(e_t)), v^g_t = W^g_V RMSNorm_E(e_t)
 * (jiphyeonjeon review §2, eq. 2.1-2.2).  Splitting a prompt over several
 * calls gives the same result as one call (§3.2).  RLT_E_CAPACITY if a row
 * would pass max_len; RLT_E_ARG if a token id is outside [0, vocab) when the
 * tokens are on the host. */
int rlt_encode(rlt_state* state, const int32_t* tokens, int n, void* stream);

/* One transition per row at t = pos_dec+1: u_t = Merge(e_t, s_{t-1})
 * (RLT-2: the register R; RLT-0: u_t = e_t), then L_D decoder blocks
 * (window self-attention over C^D, cross-attention to M_{<=t}, FFN), giving
 * H_t (greeksharifa §2.3-§2.5; jiphyeonjeon review §3).  RLT_E_ORDER if a row
 * has no encoded token at t. */
int rlt_step(rlt_state* state, void* stream);

/* T transitions per row, the recurrent prefill (jiphyeonjeon review §3.2;
 * greeksharifa App. F.1).  RLT-1 runs T sequential steps; RLT-2 runs the
 * positions of each chunk together (ceil(T/B) sequential passes when rows
 * start chunk-aligned, greeksharifa App. I.2); RLT-0 runs blocks of positions
 * together.  Same results as T calls of rlt_step. */
int rlt_prefill(rlt_state* state, int T, void* stream);

/* Readout of every row's current s_t: logits = W_out RMSNorm_out(s_t)
 * (greeksharifa §2.3).  Each output may be NULL.  logits: fp32 [batch][vocab];
 * argmax: int32 [batch], lowest index among equal maxima; sampled: int32
 * [batch], first index i with sum_{j<=i} softmax(logits/temperature)_j > u,
 * u = the SplitMix64 uniform of (rng_seed, row, rng_step):
 *   key = mix64(rng_seed ^ mix64((row+1)*G)), u = top53(mix64(key + (rng_step+1)*G))
 * with G = 0x9E3779B97F4A7C15 and mix64 the SplitMix64 finaliser.  No top-k/p
 * truncation (jiphyeonjeon review §6.2).  temperature > 0.  Each output may
 * be device or host memory; device outputs are written in stream order, host
 * outputs are valid on return (the call then synchronises `stream`). */
int rlt_readout(rlt_state* state, float* logits, int32_t* argmax, int32_t* sampled,
                uint64_t rng_seed, uint64_t rng_step, float temperature, void* stream);

/* Replay: log-probabilities of given tokens under the current weights, each
 * read from the state that precedes it, then the token is consumed
 * (jiphyeonjeon review §6.2, eq. 5.3-5.5: log pi(y|c) = sum_i log p(y_i | c,
 * y_<i); greeksharifa App. D.3, F.4).  tokens: int32 [batch][n], host or
 * device, appended to every row as by rlt_encode; then for j = 0..n-1
 *   logprobs[b][j] = log softmax(logits_b / temperature)[tokens[b][j]],
 * logits_b = W_out RMSNorm_out(s) of row b before token j is consumed (for
 * a reset row and j = 0, the readout of s_star), followed by one transition.
 * temperature = 1 is the model's own distribution; the sampler's temperature
 * gives the distribution rlt_readout samples from (same max and summation,
 * so exp(logprob) is the sampling probability up to rounding).  Afterwards
 * every row has consumed the n tokens: the same state as rlt_encode +
 * rlt_prefill(n).  A replay from the sequence start resets the rows first;
 * the prompt's terms come out beside the response's and the caller keeps the
 * ones it needs.  logprobs: fp32 [batch][n], host or device (host: valid on
 * return; the call then synchronises `stream`).  One readout and one
 * transition per position (no graph replay).  The first call allocates
 * 8 * batch * max_len bytes of scratch in the state.  Errors: RLT_E_ARG (null
 * pointers, n < 0, temperature <= 0, a host token outside [0, vocab)),
 * RLT_E_ORDER (a row has encoded tokens not yet consumed), RLT_E_CAPACITY;
 * a device token outside [0, vocab) gives NaN and RLT_E_ARG from
 * rlt_state_check. */
int rlt_replay_logprobs(rlt_state* state, const int32_t* tokens, int n, float* logprobs,
                        float temperature, void* stream);

/* Packed documents: several independent documents one after another in each
 * row.  tokens: int32 [batch][n], host or device; doc_start: uint8
 * [batch][n], HOST memory, nonzero where a document starts.  Before token j
 * of row b with doc_start[b][j] != 0 the row restarts from H_0 (as
 * rlt_state_reset: s = R = s_star, positions 0, so token j is position 1 of
 * its document): the recurrent output, window rings, encoder cache and
 * positions are per document, and no attention crosses a document start
 * (jiphyeonjeon review §6.1; greeksharifa App. F).  Every token is encoded
 * and consumed (one transition each); a row without a start at column 0
 * continues its current document.  Row b then holds the state of its last
 * document as if that document alone had been encoded and prefilled in a
 * fresh row: bit for bit for RLT-1 and RLT-0; for RLT-2 within the rounding
 * of the two schedules (a lone prefill runs each chunk's positions as one
 * block, the packed run meets chunks cut at document starts).  The columns are cut where any row starts a
 * document, and each piece is one rlt_encode + rlt_prefill for all rows, so
 * rows sit at different positions.  Synchronises `stream` at every cut.
 * Errors, checked before anything runs: RLT_E_ARG (null pointers, n < 0,
 * doc_start in device memory, a host token outside [0, vocab)), RLT_E_ORDER (a row has encoded tokens not
 * yet consumed), RLT_E_CAPACITY (a document would pass max_len); later,
 * RLT_E_DEVICE if a CUDA call fails (the rows then hold the pieces before
 * it). */
int rlt_prefill_packed(rlt_state* state, const int32_t* tokens, const uint8_t* doc_start, int n,
                       void* stream);

/* Readout of caller-supplied state vectors that allocates nothing (no
 * counterpart in the method: a serving convenience for callers that hold a
 * model but no state, and may not allocate device memory).  s_rows: device
 * fp32 [rows][d]; row r is read out exactly as rlt_readout reads out row r of
 * a state whose s_t equals it (same logits, argmax and sampled id for the
 * same rng_seed, rng_step, temperature).  Outputs as in rlt_readout: each may
 * be NULL, device or host memory; host outputs are valid on return (the call
 * then synchronises `stream`, which also ends its use of the scratch).
 * Scratch: a file-scope device array of RLT_READOUT_ROWS_SCRATCH_BYTES (16 MiB)
 * per device.  A call needs rows*d*(2 for bf16, 4 for fp32) bytes, plus
 * rows*vocab*4 when `logits` is not a device pointer, plus rows*8, each rounded
 * up to 256; a call needing more returns RLT_E_ARG and launches nothing (e.g.
 * vocab 32000, d 2048, bf16, host logits: at most 127 rows).  Nothing in the scratch
 * has to start at zero.  The first call on a device looks the array's address
 * up (cudaGetSymbolAddress), which may load the module: make that first call
 * before any stream capture on the device begins.  All calls on one device
 * share the one array: calls in flight at the same time (other streams, other
 * threads) race on it; order them on one stream.
 * RLT_E_ARG also for a null model or s_rows, s_rows not in device memory,
 * rows < 0, temperature <= 0.  rows == 0 does nothing. */
#define RLT_READOUT_ROWS_SCRATCH_BYTES (16u << 20)
int rlt_readout_rows(const rlt_model* model, const float* s_rows, int rows, float* logits,
                     int32_t* argmax, int32_t* sampled, uint64_t rng_seed, uint64_t rng_step,
                     float temperature, void* stream);

/* Host copies of the per-row positions (arrays of `batch` int32; either may
 * be NULL).  pos_enc = tokens encoded, pos_dec = transitions applied. */
int rlt_state_positions(const rlt_state* state, int32_t* pos_enc, int32_t* pos_dec);

/* Copy one state component to `dst` (host or device), `nbytes` exactly its
 * size (query with dst = NULL: *nbytes_out receives the size).  Components:
 * RLT_PART_S / _R: fp32 [batch][d]; _E: fp32 [batch][max_len][d];
 * _MEM: model dtype [batch][G][2][h][max_len][d_h]; _RING: model dtype
 * [batch][L_D][2][h][W-1][d_h]; _ENC: model dtype [batch][L_E][2][h][max_len][d_h].
 * Synchronises `stream` when dst is host memory. */
#define RLT_PART_S    0
#define RLT_PART_R    1
#define RLT_PART_E    2
#define RLT_PART_MEM  3
#define RLT_PART_RING 4
#define RLT_PART_ENC  5
int rlt_state_read(rlt_state* state, int part, void* dst, size_t nbytes, size_t* nbytes_out,
                   void* stream);

/* Exact prefix snapshot of one row: everything the row needs to continue
 * exactly as if it had never stopped -- the encoder cache C^E and memory M of
 * every encoded position, s_t (and the RLT-2 register R), the window rings
 * C^D, the encoder outputs e_t of positions not yet transitioned, pos_enc,
 * pos_dec, and the identity of the weights and config (jiphyeonjeon review
 * §6.5, multi-turn serving; greeksharifa App. E, App. H).  A row restored
 * into any state of the same model -- another row, batch size, max_len,
 * process -- continues with the same results as the row it was taken from
 * (rows are independent, see above).  New tokens (a tool's output, a user
 * turn) are appended with rlt_encode and consumed with rlt_prefill, as on the
 * original row.  The sampler keeps no state: a sampled continuation repeats
 * with the same rng_seed and rng_step.
 *
 * Snapshot bytes (little-endian), independent of batch and max_len:
 *   [0,4) "RLTS"  [4,8) u32 version 1  [8,16) u64 checksum of the weight
 *   blob's payload  [16,20) i32 pos_enc  [20,24) i32 pos_dec  [24,72) the 12
 *   int32 fields of rlt_config in declaration order  [72,96) alpha, eps,
 *   rope_base as f64  [96,128) zero;
 *   then, with P = pos_enc, h heads, d_h = d/h, G' = G if L_D > 0 else 0:
 *   s fp32 [d]; R fp32 [d]; e fp32 [P][d]; C^E [L_E][2][h][P][d_h] and
 *   M [G'][2][h][P][d_h] in the model dtype; C^D [L_D][2][h][W-1][d_h] in
 *   the model dtype (ring slot of position t: (t-1) mod (W-1)).
 * Size = 128 + 8d + 4Pd + (2 h L_E + 2 h G') P d_h e + 2 h L_D (W-1) d_h e,
 * e = 2 (bf16) or 4 (fp32).
 *
 * rlt_state_save: writes row `row`'s snapshot to `dst` (host or device),
 * `nbytes` exactly its size (query with dst = NULL: *nbytes_out receives it).
 * Ordered after the work already queued on `stream`; synchronises `stream`.
 * RLT_E_ARG for a null state, a row outside [0, batch) or a wrong nbytes.
 *
 * rlt_state_load: replaces row `row` with the snapshot at `src` (host or
 * device, `nbytes` its size); other rows are untouched.  Synchronises
 * `stream`; `src` may be freed on return.  Errors, checked before anything is
 * written: RLT_E_ARG (null state or src, bad row), RLT_E_SNAPSHOT (bad magic,
 * version or reserved bytes, nbytes not the size the header implies, or a
 * checksum or config other than the state's model), RLT_E_CAPACITY (pos_enc
 * above the state's max_len).  RLT_E_DEVICE if a copy fails: the row's
 * contents are then undefined until it is reset or loaded again.
 *
 * rlt_snapshot_info: checks a snapshot in HOST memory without a device and
 * returns its config and positions (each output may be NULL); errors as
 * rlt_state_load's format checks (RLT_E_ARG for a null snapshot). */
#define RLT_SNAPSHOT_HEADER_BYTES 128
int rlt_state_save(rlt_state* state, int row, void* dst, size_t nbytes, size_t* nbytes_out,
                   void* stream);
int rlt_state_load(rlt_state* state, int row, const void* src, size_t nbytes, void* stream);
int rlt_snapshot_info(const void* snap, size_t nbytes, rlt_config* cfg, int32_t* pos_enc,
                      int32_t* pos_dec);

/* Synchronise `stream` and report the state's sticky device error word
 * (RLT_OK, RLT_E_TIMEOUT, ...), clearing it. */
int rlt_state_check(rlt_state* state, void* stream);

/* Failure-detection self-test (no counterpart in the method).  Enqueues on
 * `stream` one small kernel whose single wait nothing will ever satisfy --
 * kind 0: an mbarrier in shared memory that no thread arrives on; kind 1: a
 * word in global memory that no thread sets -- bounded by `polls` polls
 * through the same helpers as the library's own waits.  When the wait gives
 * up the kernel records a timeout in the state's error word and returns, so
 * the next rlt_state_check reports RLT_E_TIMEOUT (and clears it) and the
 * context stays usable; the state's contents are not touched.  No copy is in
 * flight and no tensor memory is held when it gives up.  A poll of kind 0
 * lasts as long as the hardware's try-wait suspends (a system-dependent
 * limit); a poll of kind 1 sleeps about 256 ns.  RLT_E_ARG for a null state,
 * another kind, or polls outside [1, 2^24]. */
int rlt_selftest_wait(rlt_state* state, int kind, uint32_t polls, void* stream);

/* Build flags of the loaded library.  RLT_BUILD_DEBUG: built with RLT_DEBUG=1
 * (librlt_debug.so): the kernels validate every row's position counters
 * before each encoder and transition block (0 <= pos_dec, pos_dec + n <=
 * pos_enc <= max_len; pos_enc + n <= max_len when encoding), check ring
 * slots and key indices where the decode attention forms them, and token
 * ids as every build does; a violation is recorded in the state's error
 * word -- rlt_state_check then returns RLT_E_ORDER, RLT_E_CAPACITY or
 * RLT_E_ARG -- and the access it guards is skipped.  Nothing traps. */
#define RLT_BUILD_DEBUG 1u
uint32_t rlt_build_flags(void);

/* Debug builds only: overwrite the DEVICE position counters of one row,
 * leaving the host's copy unchanged -- a stand-in for a corrupted or stale
 * device state, for testing the checks above.  Synchronises `stream`.
 * Returns RLT_E_UNSUPPORTED in other builds; RLT_E_ARG for a null state or a
 * row outside [0, batch).  A counter past max_len makes the next encode write
 * past the row's buffers: only a transition or a readout may follow. */
int rlt_debug_set_positions(rlt_state* state, int row, int32_t pos_enc, int32_t pos_dec,
                            void* stream);

/* Number of kernels this library has launched in this process. */
uint64_t rlt_kernel_launches(void);

/* Live kernel timing for measurement.  While enabled (on != 0), the library
 * brackets every launch of the classes below with CUDA events recorded on the
 * launching stream and counts the algorithmic bytes each launch must move
 * (keys/values read, cache entries written, activations in and out; weights
 * excluded).  rlt_profile_query synchronises `stream`, sums the elapsed times
 * of the class since the last enable, and reports launches, total ms and
 * bytes.  Enabling resets the counters.  on = 1: transition blocks replayed
 * as CUDA graphs are timed as whole blocks (RLT_PROF_STEP) only; on = 2: they
 * replay a twin graph with event nodes around each attention launch (those
 * launches then lose their overlap with the kernel before them) and each
 * replay is followed by a stream synchronisation: for measurement only. */
#define RLT_PROF_XATTN 0  /* decoder cross-attention over M_{<=t}        */
#define RLT_PROF_SWA   1  /* decoder window attention over C^D           */
#define RLT_PROF_STEP  2  /* one whole transition block (merge .. s_t)   */
#define RLT_PROF_ENC   3  /* one whole encoder block (embed .. memory)   */
#define RLT_PROF_ENC1  4  /* the same, for a one-position call (a new   */
                          /* token during generation)                   */
#define RLT_PROF_NCLS  5
/* cls + RLT_PROF_NCLS * (l + 1) queries the window or cross-attention
 * launches of decoder layer l alone (0 <= l < L_D). */
int rlt_profile_enable(rlt_state* state, int on);
int rlt_profile_query(rlt_state* state, int cls, uint64_t* launches, double* total_ms,
                      double* bytes, void* stream);

/* Static description of a return code. */
const char* rlt_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* RLT_H */
