/*
 * prism.h -- C ABI of the Prism Attention decode hot path on B200 (sm_100a).
 *
 * Source of every operation: "Prism Attention: Proposal-Refined Index Sharing
 * Mechanism for Efficient LLMs Inference" (arXiv 2610.22985), section 4.1
 * (equations (1)-(6)) and Algorithm 1 (PrismAttention decoding at step t).
 *
 * The decode step walks a group of layers.  An anchor (proposal) layer scores
 * every cached token and keeps the exact top-kappa tokens; a refined layer
 * expands the source selection by +-r positions into a deduplicated proposal
 * set, rescores only that set with its own query and keys, and keeps its own
 * top-kappa; every layer then runs sparse GQA decode attention over its
 * kappa selected K/V rows.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named q, k, v, out, idx*, cand*, len, ws are DEVICE pointers on
 *    the current CUDA device; the caller owns every buffer.  The library
 *    allocates no device memory.  Between calls it keeps only per-device
 *    caches: the SM count, and (for prism_decode_step) four helper streams
 *    and a pool of events, created on first use and kept until exit.  These
 *    per-device caches are the library's only global state; the helper
 *    streams carry the step's multi-stream schedule.
 *  - A refined layer's selection may run inside its rescoring kernel, whose
 *    blocks of one row then wait for one another at bounded barriers; this
 *    is chosen only when the launch's blocks fit the device's SMs at once.
 *    Kernels of the caller running concurrently on other streams delay such
 *    a launch but do not change its result, unless they hold SMs for longer
 *    than the wait limit (PRISM_WAIT_LIMIT_MS, default 4000), which is then
 *    reported as PRISM_ERR_TIMEOUT in the status word.
 *  - Layouts (row-major, no padding between rows):
 *      q    bf16 [B][Hq][d]            one decode query per sequence
 *      k, v bf16 [B][Hkv][Lmax][d]     KV cache of one layer; position i of
 *                                       sequence b is row i of every head
 *      len  int32 [B]                  context length of each sequence,
 *                                       0 <= len[b] <= Lmax
 *      idx  int32 [B][Hkv][kappa]      a selection: token positions in
 *                                       ascending order, then -1 padding
 *    Query head j reads KV head j / (Hq / Hkv).
 *  - Alignment: q, k, v, out 16 bytes; int32 arrays 4 bytes; ws 256 bytes.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream), makes no host synchronisation and can be captured into
 *    a CUDA graph.  prism_decode_step forks work from `stream` onto its
 *    helper streams and joins it back before returning control of `stream`:
 *    work enqueued on `stream` afterwards sees every result.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid argument returns PRISM_ERR_INVALID_ARG (or PRISM_ERR_UNSUPPORTED
 *    for a shape the kernels do not cover, PRISM_ERR_WORKSPACE for a short
 *    workspace) and launches nothing.  A launch failure returns
 *    PRISM_ERR_CUDA.
 *  - Device-side contract violations (len[b] outside [0, Lmax], a selected
 *    index outside [0, len[b])) are clamped or skipped by the kernels, which
 *    also record the first such event in the workspace status word; a wait
 *    that runs past its time limit records PRISM_ERR_TIMEOUT there.  Read it
 *    with prism_check_device_status().
 *  - Scores are fp32 (bf16 inputs, fp32 accumulation).  Ties in a top-kappa
 *    selection go to the lower position; -0.0 ties with +0.0.
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PRISM_API __attribute__((visibility("default")))
#else
#define PRISM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PRISM_OK = 0,
    PRISM_ERR_INVALID_ARG = 1,
    PRISM_ERR_UNSUPPORTED = 2,
    PRISM_ERR_WORKSPACE = 3,
    PRISM_ERR_CUDA = 4,
    PRISM_ERR_TIMEOUT = 5,
    PRISM_ERR_DEVICE = 6
} prism_status_t;

/* Decode-step variants (Algorithm 1 and its special cases).
 * REFINE:        anchor layers select exactly (Eq. (1)-(2)); other layers
 *                expand +-radius, rescore (Eq. (5)) and reselect (Eq. (6)).
 * STATIC_REUSE:  other layers reuse the source selection unchanged (Eq. (3)).
 * DENSE_ANCHOR:  every layer is an anchor layer (per-layer exact top-kappa).
 * POOL:          the paper's proposal-refined sharing as section 4 states it:
 *                every score is the group maximum of Eq. (9),
 *                  s(i) = scale * max_{j in G(h)} <q_j, k_i>  (bf16 keys);
 *                an anchor layer keeps the pool C = TopK(s, rho * kappa) of
 *                Eq. (4) and attends to its own top-kappa (the first kappa of
 *                C in score order, Algorithm 1); every other layer rescores
 *                the nearest preceding anchor's pool with its own q and K
 *                (Eq. (5)) and keeps its top-kappa (Eq. (6)).  rho is
 *                cfg->pool_factor; radius and chain are not used. */
typedef enum {
    PRISM_MODE_REFINE = 0,
    PRISM_MODE_STATIC_REUSE = 1,
    PRISM_MODE_DENSE_ANCHOR = 2,
    PRISM_MODE_POOL = 3
} prism_mode_t;

/* Source selection of a refined layer.
 * PREV:   the previous layer's final selection (default).
 * ANCHOR: the most recent anchor layer's selection (the association f(S) of
 *         Algorithm 1). */
typedef enum {
    PRISM_CHAIN_PREV = 0,
    PRISM_CHAIN_ANCHOR = 1
} prism_chain_t;

/* Shape and policy of one decode step.  All fields are plain int32/float so
 * that the struct has the same layout from C, C++ and Python (ctypes). */
typedef struct {
    int32_t batch;          /* B >= 1                                         */
    int32_t n_q_heads;      /* Hq >= 1                                        */
    int32_t n_kv_heads;     /* Hkv >= 1, Hq % Hkv == 0, G = Hq/Hkv in {1,2,4,8,16} */
    int32_t head_dim;       /* d in {64, 128}                                 */
    int32_t max_len;        /* Lmax, 1 <= Lmax <= PRISM_MAX_LEN               */
    int32_t kappa;          /* sparse budget, 1 <= kappa <= PRISM_MAX_LEN     */
    int32_t radius;         /* proposal radius r >= 0                         */
    int32_t n_layers;       /* N >= 1 for prism_decode_step, <= PRISM_MAX_LAYERS */
    const uint8_t *anchor_mask; /* HOST array [N] of layer kinds (Table 9's F/R/S):
                                   1 = anchor (F), 0 = refined (R; a reuse layer
                                   in STATIC_REUSE), 2 = shared (S: keeps the
                                   previous layer's selection, i.e. that of the
                                   nearest preceding F or R layer, with no
                                   rescoring); other values are invalid.
                                   mask[0] must be 1 unless DENSE_ANCHOR, which
                                   ignores the array.  prism_decode_step only;
                                   may be NULL for the single-stage calls.    */
    int32_t mode;           /* prism_mode_t                                   */
    int32_t chain;          /* prism_chain_t                                  */
    float scale;            /* score/logit scale; 0 means 1/sqrt(d)           */
    int32_t flags;          /* PRISM_FLAG_* bits, 0 by default                */
    int32_t pool_factor;    /* rho >= 1 with rho * kappa <= PRISM_MAX_LEN in
                               PRISM_MODE_POOL; ignored by the other modes    */
} prism_config_t;

/* prism_decode_step schedules anchor scoring, selections and attention as a
 * DAG over helper streams; this flag enqueues everything, in layer order, on
 * the caller's stream instead (same results, bit for bit). */
#define PRISM_FLAG_SERIAL 1
/* PRISM_MODE_POOL only: the proposal scores (Eq. (9)) use 2-bit keys
 * (section 4.2, Eq. (7)-(8)).  With this flag the `k` argument of
 * prism_index_anchor, prism_index_pool, prism_score_anchor and
 * prism_index_refine is a 2-bit key cache written by prism_quantize_keys,
 * and the decode step is prism_decode_step_kq (bf16 keys for attention, the
 * 2-bit cache for scoring); prism_decode_step rejects the flag. */
#define PRISM_FLAG_INT2_KEYS 2

#define PRISM_MAX_LEN (1 << 20)
#define PRISM_MAX_BATCH_ROWS 65535   /* B * Hkv */
#define PRISM_MAX_LAYERS 4096

/* Bytes of workspace every call below needs for `cfg` (the same figure serves
 * all of them; it grows with n_layers, which the single-stage calls may leave
 * at 0 or 1).  The workspace holds scores, candidate lists, histograms,
 * selections and attention partials; its first 256 bytes are the device
 * status word.  Pass it 256-byte aligned.  Zero the status word (the first
 * 256 bytes) once after allocating the workspace, e.g. by allocating it
 * zero-filled; the rest needs no initialisation and is scratch between
 * calls.  The status word persists across calls until
 * prism_check_device_status() reads and clears it.
 * Errors: PRISM_ERR_INVALID_ARG / PRISM_ERR_UNSUPPORTED for a bad config. */
PRISM_API prism_status_t prism_workspace_size(const prism_config_t *cfg, size_t *bytes);

/* Anchor layer index construction: Eq. (1) over every cached token, then the
 * exact top-kappa of Eq. (2).
 *   s[b][h][i] = scale * sum_{j in G(h)} <q[b][j], k[b][h][i]>, i < len[b]
 *                (PRISM_MODE_POOL: scale * max_{j in G(h)} <q[b][j], k[b][h][i]>,
 *                Eq. (9))
 *   idx_out[b][h] = the min(kappa, len[b]) positions with the largest s,
 *                   ties to the lower position, ascending, -1 padded.
 * q          bf16 [B][Hq][d]           k bf16 [B][Hkv][Lmax][d]
 * len        int32 [B]                 idx_out int32 [B][Hkv][kappa] (written)
 * scores_out fp32 [B][Hkv][Lmax] or NULL; when given, receives s (entries at
 *            i >= len[b] are left untouched).                                */
PRISM_API prism_status_t prism_index_anchor(const prism_config_t *cfg, const void *q,
                                  const void *k, const int32_t *len,
                                  int32_t *idx_out, float *scores_out,
                                  void *ws, size_t ws_bytes, void *stream);

/* Proposal layer of PRISM_MODE_POOL (cfg->mode must be PRISM_MODE_POOL):
 * the group-maximum scores of Eq. (9) over every cached token, the candidate
 * pool of Eq. (4) and the layer's own selection (Algorithm 1, proposal
 * branch).
 *   s[b][h][i]     = scale * max_{j in G(h)} <q[b][j], k[b][h][i]>, i < len[b]
 *   pool_out[b][h] = the min(rho*kappa, len[b]) positions with the largest s
 *                    (Eq. (4), rho = cfg->pool_factor), ascending, -1 padded
 *   idx_out[b][h]  = the first kappa of the pool in score order, i.e. the
 *                    min(kappa, len[b]) largest s, ascending, -1 padded
 * Ties go to the lower position in both.
 * pool_out   int32 [B][Hkv][rho*kappa] (written)
 * idx_out    int32 [B][Hkv][kappa] (written)
 * scores_out fp32 [B][Hkv][Lmax] or NULL (as for prism_index_anchor).        */
PRISM_API prism_status_t prism_index_pool(const prism_config_t *cfg, const void *q,
                                  const void *k, const int32_t *len,
                                  int32_t *pool_out, int32_t *idx_out,
                                  float *scores_out, void *ws, size_t ws_bytes,
                                  void *stream);

/* Anchor scoring only: Eq. (1) over every cached token, exactly one kernel
 * launch (the streaming kernel that prism_index_anchor starts with).  Meant
 * for timing that kernel on its own and for diagnostics.
 * scores_out fp32 [B][Hkv][Lmax] (written for i < len[b]).  The first-digit
 * histogram region of the workspace is accumulated, not reset, by this call;
 * the other calls reset it before use. */
PRISM_API prism_status_t prism_score_anchor(const prism_config_t *cfg, const void *q,
                                  const void *k, const int32_t *len,
                                  float *scores_out, void *ws, size_t ws_bytes,
                                  void *stream);

/* Refined layer index refinement: proposal P = { p : |p - i| <= radius for
 * some i in idx_prev[b][h], 0 <= p < len[b] } (a set, so duplicates vanish);
 * the scores of Eq. (5) on P only, with this layer's q and k; then the
 * top-kappa of Eq. (6) over P, same tie and order rules as the anchor.
 * idx_prev   int32 [B][Hkv][kappa]: entries < 0 are padding and skipped; any
 *            order is accepted.
 * idx_out    int32 [B][Hkv][kappa] (written; may not alias idx_prev).
 * In PRISM_MODE_POOL the candidate set is the pool itself (Eq. (5)) and the
 * scores are the group maximum of Eq. (9): idx_prev is then a pool, int32
 * [B][Hkv][rho*kappa] (any order, duplicates and -1 padding allowed), and
 * radius is not used.
 * cand_pos, cand_score, cand_count: optional diagnostic copies of P (all
 *            three NULL, or all three given): cand_pos int32 [B][Hkv][cand_cap]
 *            ascending positions, cand_score fp32 [B][Hkv][cand_cap] their
 *            scores, cand_count int32 [B][Hkv] = |P| (entries beyond
 *            cand_cap are not stored).                                       */
PRISM_API prism_status_t prism_index_refine(const prism_config_t *cfg, const void *q,
                                  const void *k, const int32_t *len,
                                  const int32_t *idx_prev, int32_t *idx_out,
                                  int32_t *cand_pos, float *cand_score,
                                  int32_t *cand_count, int32_t cand_cap,
                                  void *ws, size_t ws_bytes, void *stream);

/* Sparse GQA decode attention (the SparseAttn step of Algorithm 1): for every
 * query head j of KV head h,
 *   z_i = scale * <q[b][j], k[b][h][i]>,  i in idx[b][h] (entries < 0 skipped)
 *   out[b][j] = sum_i softmax(z)_i * v[b][h][i]   (0 if nothing is selected)
 * computed split-K with an online softmax and a final combine.
 * idx   int32 [B][Hkv][n_idx], 1 <= n_idx <= kappa   out bf16 [B][Hq][d]     */
PRISM_API prism_status_t prism_sparse_decode(const prism_config_t *cfg, const void *q,
                                   const void *k, const void *v,
                                   const int32_t *len, const int32_t *idx,
                                   int32_t n_idx, void *out, void *ws,
                                   size_t ws_bytes, void *stream);

/* prism_sparse_decode without a caller workspace.  The paper has no
 * counterpart: this is a library convenience for callers that cannot provide
 * device scratch (a host holding only device pointers to its KV cache, with
 * no device allocator of its own, or one that must not allocate once it has
 * started).  Same computation, arguments and validation as
 * prism_sparse_decode; the split-K scratch is a fixed device array inside the
 * library, so nothing is allocated by this call or by the library.
 * Limits (else PRISM_ERR_WORKSPACE, nothing launched):
 *   B * Hkv <= 1024  and  B * Hkv * ceil(n_idx / 64) * G * head_dim <= 2^20.
 * The first call on a device looks up the array's address; make it before any
 * stream capture.  All calls share the one array: calls that overlap in time
 * (other streams, other threads) race on it and must be serialised by the
 * caller.  Device-side contract violations (len outside [0, Lmax]) are
 * clamped as in prism_sparse_decode but not reported.                        */
PRISM_API prism_status_t prism_sparse_decode_noalloc(const prism_config_t *cfg, const void *q,
                                   const void *k, const void *v,
                                   const int32_t *len, const int32_t *idx,
                                   int32_t n_idx, void *out, void *stream);

/* One decode step over cfg->n_layers layers (Algorithm 1), per cfg->mode and
 * cfg->chain, every layer ending in sparse attention over its own selection.
 * q        bf16 [N][B][Hq][d] (device)
 * k, v     HOST arrays of N device pointers, each bf16 [B][Hkv][Lmax][d]
 * len      int32 [B] (device)
 * out      bf16 [N][B][Hq][d] (written)
 * idx_out  int32 [N][B][Hkv][kappa] or NULL: every layer's selection.        */
PRISM_API prism_status_t prism_decode_step(const prism_config_t *cfg, const void *q,
                                 const void *const *k, const void *const *v,
                                 const int32_t *len, void *out,
                                 int32_t *idx_out, void *ws, size_t ws_bytes,
                                 void *stream);

/* The 2-bit proposal key cache of one layer (section 4.2, Eq. (7)-(8)):
 * every key row is split into groups of 32 elements; group m keeps
 *   alpha_m = (max - min) / 3,  beta_m = min  (fp32),
 *   code_e  = clip(round half up((k_e - beta_m) / alpha_m), 0, 3),
 * alpha_m = 0 giving code 0, each an IEEE binary32 operation.  Positions
 * [start, len[b]) of every (batch, KV head) are (re)written -- the
 * append-time use quantizes the newly appended tokens -- the rest of kq is
 * left untouched.
 * k   bf16 [B][Hkv][Lmax][d] (d in {64, 128})
 * kq  uint8 [B][Hkv][Lmax][d/2]: per row, d/4 bytes of codes (byte
 *     t*(d/16) + kk holds the codes of elements 16kk + 2t, 16kk + 2t + 1,
 *     16kk + 2t + 8, 16kk + 2t + 9 in bits 0-1, 2-3, 4-5, 6-7; t = 0..3,
 *     kk = 0..d/16-1), then alpha_m, beta_m (fp32) for each group m.
 * ws  only its status word is used (a len[b] outside [0, Lmax] is
 *     recorded there).  No other field of cfg than its shape is read. */
PRISM_API prism_status_t prism_quantize_keys(const prism_config_t *cfg, const void *k,
                                   const int32_t *len, int32_t start, void *kq,
                                   void *ws, size_t ws_bytes, void *stream);

/* prism_decode_step with 2-bit proposal keys: cfg->mode == PRISM_MODE_POOL
 * and cfg->flags has PRISM_FLAG_INT2_KEYS.  kq: HOST array of N device
 * pointers, each layer's 2-bit cache (prism_quantize_keys); the anchor scans
 * and the pool rescoring read kq (Algorithm 1: INT2 keys in proposal and
 * refinement), the sparse attention reads k and v. */
PRISM_API prism_status_t prism_decode_step_kq(const prism_config_t *cfg, const void *q,
                                    const void *const *k, const void *const *v,
                                    const void *const *kq, const int32_t *len,
                                    void *out, int32_t *idx_out, void *ws,
                                    size_t ws_bytes, void *stream);

/* Synchronises `stream`, reads the workspace status word and clears it.
 * Returns PRISM_OK, PRISM_ERR_TIMEOUT (a bounded wait ran out) or
 * PRISM_ERR_DEVICE (a device-side contract violation); `detail` (nullable)
 * receives {code, where, value, 0}. */
PRISM_API prism_status_t prism_check_device_status(void *ws, size_t ws_bytes,
                                         void *stream, uint32_t detail[4]);

/* Test hook for the bounded waits: launches one CTA that waits on a barrier
 * nothing will complete, for at most `limit_ns` nanoseconds, then records
 * PRISM_ERR_TIMEOUT in the status word and returns.  It never hangs. */
PRISM_API prism_status_t prism_debug_wait_timeout(void *ws, size_t ws_bytes,
                                        uint64_t limit_ns, void *stream);

/* Static, human-readable name of a status code. */
PRISM_API const char *prism_status_string(prism_status_t status);

/* Number of kernels the calling host thread has launched through this
 * library since it was loaded (memsets and copies excluded). */
PRISM_API uint64_t prism_launch_count(void);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
PRISM_API int32_t prism_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H */
