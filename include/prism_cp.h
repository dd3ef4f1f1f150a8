/*
 * prism_cp.h -- context-parallel form of the Prism Attention decode step:
 * one long sequence split by position across ranks (one GPU each).
 *
 * Source of the operations: "Prism Attention: Proposal-Refined Index Sharing
 * Mechanism for Efficient LLMs Inference", section 4.1 (Eq. (1)-(6)),
 * section 4.2 (Eq. (4), (9): the pool variant) and Algorithm 1.  The paper
 * itself times its kernels at the shapes of one tensor-parallel rank (TP8: one
 * KV head per GPU; Appendix D, per-layer timing under the SGLang integration);
 * splitting the context is this library's own extension for contexts whose
 * KV cache outgrows one GPU.  It changes no result:
 *
 *  - Exact distributed top-k.  Order tokens by (score descending, position
 *    ascending).  A token among the k first of the whole sequence is among
 *    the k first of its own shard, so the k first of the union of every
 *    shard's k first are the k first of the sequence (Eq. (2), (4), (6)).
 *    prism_cp_index_local gives a shard's k first with their scores;
 *    prism_cp_merge selects from all shards' lists, gathered by the caller.
 *  - Split softmax.  Attention over a selection T (Algorithm 1, SparseAttn)
 *    is the merge of partial results over T ∩ shard: per query head the
 *    running maximum m, the sum l of exp(z - m) and the accumulator
 *    acc = sum exp(z - m) v; o = sum_r e^(m_r - M) acc_r / sum_r e^(m_r - M) l_r
 *    with M = max_r m_r.  prism_cp_attn_local gives a shard's (acc, m, l);
 *    prism_cp_combine merges all shards' partials, gathered by the caller.
 *
 * The exchange between the two halves of each step (an all-gather of a few
 * hundred KB per layer) is the caller's: the Python layer uses
 * torch.distributed over NCCL.
 *
 * Sharding.  Rank r of R holds the global positions
 * [r * shard_len, (r + 1) * shard_len) of every sequence and KV head: its K
 * and V buffers are bf16 [B][Hkv][shard_len][d], row i holding global
 * position r * shard_len + i.  cfg->max_len is the global capacity, at most
 * R * shard_len; len is the GLOBAL length array (device int32 [B]).  A shard
 * past a sequence's end holds no token of it.
 *
 * Conventions are those of prism.h (device pointers, caller-owned buffers,
 * host-side validation before any launch, asynchronous on `stream`, graph
 * capturable, device-side violations recorded in the workspace status word).
 * The workspace is sized by prism_cp_workspace_size for (cfg, shard) and is
 * shared by all four calls of a rank; it must not be used by two calls in
 * flight at the same time.  Supported: modes PRISM_MODE_REFINE,
 * PRISM_MODE_STATIC_REUSE, PRISM_MODE_DENSE_ANCHOR and PRISM_MODE_POOL on
 * bf16 keys (PRISM_FLAG_INT2_KEYS returns PRISM_ERR_UNSUPPORTED).
 */
#ifndef PRISM_CP_H
#define PRISM_CP_H

#include "prism.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t n_ranks;    /* R >= 1 */
    int32_t rank;       /* 0 <= rank < R */
    int32_t shard_len;  /* positions per shard, >= 1; R * shard_len >= cfg->max_len */
} prism_cp_shard_t;

/* Workspace bytes of one rank for (cfg, shard). */
PRISM_API prism_status_t prism_cp_workspace_size(const prism_config_t *cfg,
                                                 const prism_cp_shard_t *shard, size_t *bytes);

/* This shard's half of a selection (Eq. (2) for an anchor layer, Eq. (5)-(6)
 * for a refined one).
 *  src == NULL: anchor layer.  Every token of the shard is scored (Eq. (1);
 *    in pool mode the group maximum of Eq. (9)) and the shard's k first are
 *    kept.  In pool mode the shard's rho*kappa first (the pool of Eq. (4))
 *    also go to pool_pos/pool_score, which are required then and must be
 *    NULL otherwise.
 *  src != NULL: refined layer.  src is the canonical GLOBAL source selection
 *    (int32 [B][Hkv][s], ascending positions then -1 padding, as
 *    prism_cp_merge writes it; s = kappa, or rho*kappa in pool mode).  The
 *    proposal (every position within cfg->radius of a source token, clipped
 *    to [0, len[b]); radius 0 in pool mode) is intersected with the shard,
 *    rescored with this layer's q and K, and the shard's kappa first kept.
 * Output cand_pos int32 [B][Hkv][kappa]: GLOBAL positions, ascending, then -1
 * padding; cand_score fp32 [B][Hkv][kappa]: their scores (Eq. (1) scale
 * included), -inf at padding.  pool_pos/pool_score: the same with rho*kappa
 * entries.  q: bf16 [B][Hq][d]; k: this shard's keys. */
PRISM_API prism_status_t prism_cp_index_local(const prism_config_t *cfg,
                                              const prism_cp_shard_t *shard, const void *q,
                                              const void *k, const int32_t *len,
                                              const int32_t *src, int32_t *cand_pos,
                                              float *cand_score, int32_t *pool_pos,
                                              float *pool_score, void *ws, size_t ws_bytes,
                                              void *stream);

/* Exact top-n_out over the gathered per-shard lists: cand_pos/cand_score
 * [n_ranks][B][Hkv][n_out] (shard r's list at r; each list ascending then -1
 * padding, as prism_cp_index_local writes it).  n_out is kappa (a
 * selection) or, in pool mode, rho*kappa (a pool).  idx_out int32
 * [B][Hkv][n_out]: ascending global positions, min(n_out, len[b]) of them,
 * then -1 padding.  Ties go to the lower position.  ws: a workspace of
 * prism_cp_workspace_size for any shard of the same n_ranks. */
PRISM_API prism_status_t prism_cp_merge(const prism_config_t *cfg,
                                        const prism_cp_shard_t *shard, int32_t n_out,
                                        const int32_t *cand_pos, const float *cand_score,
                                        const int32_t *len, int32_t *idx_out, void *ws,
                                        size_t ws_bytes, void *stream);

/* This shard's partial of the sparse GQA attention over the global
 * selection idx (int32 [B][Hkv][kappa], ascending global positions then -1
 * padding; any entry may lie in another shard).  part_out fp32
 * [B][Hq][d + 2]: per query head the unnormalised accumulator acc[d], then
 * m and l (m = -inf, l = 0, acc = 0 when no selected token lies in this
 * shard).  k, v: this shard's K and V. */
PRISM_API prism_status_t prism_cp_attn_local(const prism_config_t *cfg,
                                             const prism_cp_shard_t *shard, const void *q,
                                             const void *k, const void *v, const int32_t *len,
                                             const int32_t *idx, float *part_out, void *ws,
                                             size_t ws_bytes, void *stream);

/* Merge of the gathered partials part_all fp32 [n_ranks][B][Hq][d + 2]
 * into out bf16 [B][Hq][d] (zeros for a head with no selected token). */
PRISM_API prism_status_t prism_cp_combine(const prism_config_t *cfg, int32_t n_ranks,
                                          const float *part_all, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_CP_H */
