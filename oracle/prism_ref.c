/*
 * prism_ref.c -- the ORACLE for the Prism Attention decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, obviously correct CPU
 * statement of what the decode step computes.  It is called only by the test
 * suite, by the smoke check and by the CPU-baseline leg of the benchmark.  The
 * CUDA library never links, includes or calls it, and it shares no code with
 * the CUDA library.
 *
 * Source: "Prism Attention: Proposal-Refined Index Sharing Mechanism for
 * Efficient LLMs Inference" (arXiv 2610.22985), section 4.1, equations (1)-(6),
 * and Algorithm 1 (PrismAttention decoding at step t).
 *
 * Variant implemented (where the paper leaves a step open, the plainest
 * reading that the rest of it supports):
 *   - relevance score phi(q, k_i) = scale * sum_{j in G(h)} <q_j, k_i> on the
 *     bf16 key cache, accumulated in fp64 (Eq. (1));
 *   - TopK returns the kappa largest scores, ties broken by the lower token
 *     position, the result listed in ascending position order (Eq. (2), (6));
 *   - a refined layer rescores a proposal set made of every position within
 *     +-r of a previously selected index, clipped to [0, L) (Eq. (5) over the
 *     positional proposal), and reselects its own top-kappa (Eq. (6));
 *   - sparse attention over the selected rows with an exact softmax (the
 *     SparseAttn step of Algorithm 1);
 *   - the 2-bit proposal keys of section 4.2 (Eq. (7)-(9)) for mode 3;
 *   - the pool variant (mode 3) of section 4.1-4.2 as the paper states it:
 *     the relevance score is the maximum over the GQA group (Eq. (9), on the
 *     bf16 keys), an anchor layer keeps a pool of the rho*kappa best tokens
 *     (Eq. (4)) and attends to the first kappa of that pool in score order
 *     (Algorithm 1, proposal-layer branch), and every refined layer rescores
 *     the most recent anchor's pool with its own q and K (Eq. (5)) and keeps
 *     its top-kappa (Eq. (6)).
 *
 * Inputs are raw bf16 bit patterns (uint16); every product and sum is formed
 * in double precision.  There is no blocking, fusion or reordering beyond the
 * definitions.
 *
 * PRISM_REF_PLANT (compile-time, default 0) plants one deliberate mistake; the
 * test suite builds those variants to show that its pins catch each of them.
 *
 * Parity pins: every function here is pinned by tests/test_oracle.py (brute
 * force, library routines, closed forms and hand cases in tests/golden/).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef PRISM_REF_PLANT
#define PRISM_REF_PLANT 0
#endif

/* Group size g of the 2-bit proposal keys (Eq. (7); the paper leaves g open). */
#define PRISM_REF_QGROUP 32

/* bf16 is the top half of an IEEE-754 binary32; widening to double is exact. */
static double bf16_to_double(uint16_t h)
{
#if PRISM_REF_PLANT == 9
    uint32_t u = (uint32_t)h << 15;            /* planted: wrong bit position */
#else
    uint32_t u = (uint32_t)h << 16;
#endif
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int prism_ref_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the row-parallel loops from now on (n >= 1); for timing only. */
void prism_ref_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int prism_ref_plant(void) { return PRISM_REF_PLANT; }

/*
 * Relevance score, Eq. (1): s(i) = phi(q, k_i) for every listed position.
 * phi(q, k) = scale * sum over the query heads j of the GQA group of <q_j, k>.
 *
 * q_group : [G][d] bf16 bits, the query heads that share this KV head
 * k_rows  : [*][d] bf16 bits, the key cache of this (batch, KV head)
 * pos     : n positions to score; NULL scores positions 0..n-1
 * s_out   : [n] fp64 scores, s_out[e] belongs to position pos[e]
 */
void prism_ref_score(int d, int G, const uint16_t *q_group,
                     const uint16_t *k_rows, int n, const int32_t *pos,
                     double scale, double *s_out)
{
    int g_used = G;
#if PRISM_REF_PLANT == 1
    if (G > 1) g_used = G - 1;                 /* planted: drops one head */
#endif
    for (int e = 0; e < n; ++e) {
        long i = pos ? (long)pos[e] : (long)e;
        double acc = 0.0;
        for (int j = 0; j < g_used; ++j) {
            for (int c = 0; c < d; ++c) {
#if PRISM_REF_PLANT == 8
                /* planted: transposed operand (key read column-major) */
                double kv = bf16_to_double(k_rows[(size_t)c * (size_t)n + (size_t)i]);
#else
                double kv = bf16_to_double(k_rows[(size_t)i * (size_t)d + (size_t)c]);
#endif
                acc += bf16_to_double(q_group[(size_t)j * (size_t)d + (size_t)c]) * kv;
            }
        }
        s_out[e] = scale * acc;
    }
}

/*
 * Proposal score of Eq. (9) on the bf16 key cache:
 *   s(i) = scale * max over the query heads j of the GQA group of <q_j, k_i>.
 * (Eq. (9) has no scale; a positive scale does not change any selection and
 * keeps the values comparable with Eq. (1).)  Arguments as prism_ref_score.
 */
void prism_ref_score_max(int d, int G, const uint16_t *q_group,
                         const uint16_t *k_rows, int n, const int32_t *pos,
                         double scale, double *s_out)
{
    for (int e = 0; e < n; ++e) {
        long i = pos ? (long)pos[e] : (long)e;
        const uint16_t *kr = k_rows + (size_t)i * (size_t)d;
        double best = -INFINITY;
        for (int j = 0; j < G; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += bf16_to_double(q_group[(size_t)j * (size_t)d + (size_t)c]) *
                       bf16_to_double(kr[c]);
#if PRISM_REF_PLANT == 12
            best = (j == 0) ? dot : best + dot;    /* planted: sum instead of max */
#else
            if (dot > best) best = dot;
#endif
        }
        s_out[e] = scale * best;
    }
}

/*
 * Group-wise asymmetric b = 2 bit quantization of one key row, Eq. (7)-(8):
 * the d elements split into d/g groups of g; group m keeps
 *   alpha_m = (max - min) / (2^b - 1),  beta_m = min,
 *   code_e  = clip(round((k_e - beta_m) / alpha_m), 0, 3)  (round half up),
 * and alpha_m = 0 (all codes 0) when max == min.  Every step is an IEEE
 * binary32 operation (the codes are decided in the kernel's precision).
 * codes: [d] one code per element; alpha, beta: [d/g].
 */
void prism_ref_quantize_row(int d, int g, const uint16_t *k_row, uint8_t *codes, float *alpha,
                            float *beta)
{
    for (int m = 0; m < d / g; ++m) {
        float lo = (float)bf16_to_double(k_row[m * g]), hi = lo;
        for (int e = 1; e < g; ++e) {
            const float x = (float)bf16_to_double(k_row[m * g + e]);
            if (x < lo) lo = x;
            if (x > hi) hi = x;
        }
#if PRISM_REF_PLANT == 17
        volatile float a = (hi - lo) / 4.0f;        /* planted: 2^b levels, not 2^b - 1 */
#else
        volatile float a = (hi - lo) / 3.0f;
#endif
        alpha[m] = a;
        beta[m] = lo;
        for (int e = 0; e < g; ++e) {
            int c = 0;
            if (a > 0.0f) {
                volatile float t = (float)bf16_to_double(k_row[m * g + e]) - lo;
                volatile float x = t / a;
#if PRISM_REF_PLANT == 18
                c = (int)floorf(x);                     /* planted: truncation, not rounding */
#else
                volatile float xr = x + 0.5f;
                c = (int)floorf(xr);
#endif
                if (c < 0) c = 0;
                if (c > 3) c = 3;
            }
            codes[m * g + e] = (uint8_t)c;
        }
    }
}

/*
 * Proposal score of Eq. (9) on the 2-bit keys: the group maximum of
 * <q_j, khat_i> with khat_i,e = alpha_m * code_e + beta_m (the dequantized
 * key; group m holds element e), times scale, in fp64.
 * codes: [*][d] (one per element), alpha/beta: [*][d/g]; pos as prism_ref_score.
 */
void prism_ref_score_max_q2(int d, int g, int G, const uint16_t *q_group, const uint8_t *codes,
                            const float *alpha, const float *beta, int n, const int32_t *pos,
                            double scale, double *s_out)
{
    const int M = d / g;
    for (int e = 0; e < n; ++e) {
        long i = pos ? (long)pos[e] : (long)e;
        double best = -INFINITY;
        for (int j = 0; j < G; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) {
                const int m = c / g;
#if PRISM_REF_PLANT == 19
                const double kh = (double)alpha[i * M + m] * codes[(size_t)i * d + c];   /* planted: beta dropped */
#else
                const double kh = (double)alpha[i * M + m] * codes[(size_t)i * d + c] +
                                  (double)beta[i * M + m];
#endif
                dot += bf16_to_double(q_group[(size_t)j * (size_t)d + (size_t)c]) * kh;
            }
            if (dot > best) best = dot;
        }
        s_out[e] = scale * best;
    }
}

typedef struct {
    double s;
    int32_t p;
} ref_item_t;

/* Order of Eq. (2): larger score first; equal scores, lower position first. */
static int ref_item_cmp(const void *a, const void *b)
{
    const ref_item_t *x = (const ref_item_t *)a;
    const ref_item_t *y = (const ref_item_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
#if PRISM_REF_PLANT == 2
    return (x->p > y->p) ? -1 : (x->p < y->p) ? 1 : 0;   /* planted: higher wins */
#else
    return (x->p < y->p) ? -1 : (x->p > y->p) ? 1 : 0;
#endif
}

static int ref_int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x < y) ? -1 : (x > y) ? 1 : 0;
}

/*
 * TopK, Eq. (2) and Eq. (6): the positions of the kappa largest scores.
 * Sorts (score descending, position ascending) and keeps the first
 * min(kappa, n); the kept positions are then listed in ascending order and
 * out[kappa_eff..kappa) is filled with -1.  -0.0 and +0.0 compare equal, so
 * they tie and the lower position wins.  Returns kappa_eff.
 */
int prism_ref_topk(int n, const double *s, const int32_t *pos, int kappa,
                   int32_t *out)
{
    int keff = n < kappa ? n : kappa;
#if PRISM_REF_PLANT == 3
    if (keff > 1 && keff == kappa) keff -= 1;  /* planted: off-by-one budget */
#endif
    ref_item_t *it = (ref_item_t *)malloc(sizeof(ref_item_t) * (size_t)(n > 0 ? n : 1));
    for (int e = 0; e < n; ++e) {
        it[e].s = s[e];
        it[e].p = pos ? pos[e] : e;
    }
    qsort(it, (size_t)n, sizeof(ref_item_t), ref_item_cmp);
    for (int t = 0; t < keff; ++t) out[t] = it[t].p;
    qsort(out, (size_t)keff, sizeof(int32_t), ref_int_cmp);
    for (int t = keff; t < kappa; ++t) out[t] = -1;
    free(it);
    return keff;
}

/*
 * Positional proposal set: every position p with |p - i| <= r for some
 * previously selected index i, clipped to [0, L).  A set, so duplicates
 * vanish.  Entries of idx_prev that are negative (padding) or >= L are
 * ignored.  Writes the positions in ascending order and returns |P|.
 */
int prism_ref_expand(int L, int n_prev, const int32_t *idx_prev, int r,
                     int32_t *pos_out)
{
    if (L <= 0) return 0;
    unsigned char *mark = (unsigned char *)calloc((size_t)L, 1);
    for (int t = 0; t < n_prev; ++t) {
        long i = idx_prev[t];
        if (i < 0 || i >= L) continue;
#if PRISM_REF_PLANT == 4
        long lo = i - (long)r + 1;             /* planted: window one short */
#else
        long lo = i - (long)r;
#endif
        long hi = i + (long)r;
        if (lo < 0) lo = 0;
        if (hi > L - 1) hi = L - 1;
        for (long p = lo; p <= hi; ++p) mark[p] = 1;
    }
    int n = 0;
    for (int p = 0; p < L; ++p)
        if (mark[p]) pos_out[n++] = p;
    free(mark);
    return n;
}

/*
 * Sparse attention of one GQA group over an index set (the SparseAttn step of
 * Algorithm 1): for each query head j of the group,
 *   z_i = scale * <q_j, k_i>  for i in T,
 *   p_i = exp(z_i - max z) / sum_i' exp(z_i' - max z),
 *   o_j = sum_i p_i v_i.
 * idx entries < 0 are padding.  An empty set gives o_j = 0 and weight sum 0.
 * wsum (nullable) receives sum_i p_i per head.
 */
void prism_ref_attention(int d, int G, const uint16_t *q_group,
                         const uint16_t *k_rows, const uint16_t *v_rows,
                         int n_idx, const int32_t *idx, double scale,
                         double *out, double *wsum)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)(n_idx > 0 ? n_idx : 1));
    for (int j = 0; j < G; ++j) {
        const uint16_t *qj = q_group + (size_t)j * (size_t)d;
        double zmax = -INFINITY;
        int nvalid = 0;
        for (int t = 0; t < n_idx; ++t) {
            if (idx[t] < 0) continue;
            const uint16_t *kr = k_rows + (size_t)idx[t] * (size_t)d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += bf16_to_double(qj[c]) * bf16_to_double(kr[c]);
#if PRISM_REF_PLANT == 5
            z[t] = acc;                        /* planted: scale dropped */
#else
            z[t] = scale * acc;
#endif
            if (z[t] > zmax) zmax = z[t];
            ++nvalid;
        }
        double *oj = out + (size_t)j * (size_t)d;
        for (int c = 0; c < d; ++c) oj[c] = 0.0;
        if (nvalid == 0) {
            if (wsum) wsum[j] = 0.0;
            continue;
        }
        double l = 0.0;
        for (int t = 0; t < n_idx; ++t) {
            if (idx[t] < 0) continue;
            l += exp(z[t] - zmax);
        }
        double wtot = 0.0;
        for (int t = 0; t < n_idx; ++t) {
            if (idx[t] < 0) continue;
#if PRISM_REF_PLANT == 7
            double p = exp(z[t] - zmax);       /* planted: not normalised */
#else
            double p = exp(z[t] - zmax) / l;
#endif
            wtot += p;
#if PRISM_REF_PLANT == 6
            const uint16_t *vr = k_rows + (size_t)idx[t] * (size_t)d;   /* planted: K for V */
#else
            const uint16_t *vr = v_rows + (size_t)idx[t] * (size_t)d;
#endif
            for (int c = 0; c < d; ++c) oj[c] += p * bf16_to_double(vr[c]);
        }
        if (wsum) wsum[j] = wtot;
    }
    free(z);
}

/*
 * One decode step over n_layers layers, following Algorithm 1.
 *
 * mode 0 (refine):        an anchor layer scores every cached token (Eq. (1))
 *                         and keeps its exact top-kappa (Eq. (2)); any other
 *                         layer expands the source selection by +-r, rescores
 *                         only that proposal with its own q and K (Eq. (5))
 *                         and reselects top-kappa (Eq. (6)).
 * mode 1 (static reuse):  a non-anchor layer copies the source selection
 *                         (Eq. (3)).
 * mode 2 (dense anchor):  every layer is an anchor layer.
 * mode 3 (pool):          scores are the group maximum of Eq. (9); an anchor
 *                         layer keeps the pool C = TopK(s, rho*kappa) of
 *                         Eq. (4) and selects the first kappa tokens of C in
 *                         score order; any other layer rescores the most
 *                         recent anchor's pool with its own q and K (Eq. (5))
 *                         and keeps its top-kappa (Eq. (6)).  r and chain are
 *                         not used: the association f(S) of Algorithm 1 is
 *                         the nearest preceding anchor.
 * chain 0: the source selection is the previous layer's final selection.
 * chain 1: the source selection is the most recent anchor layer's selection
 *          (the anchor-rooted association f(S) of Algorithm 1).
 * Layer kinds (anchor_mask[l], ignored in mode 2): 1 = anchor (F), 0 = the
 * mode's other layer (R: refined; static reuse in mode 1), 2 = shared (S,
 * Table 9): the layer keeps the previous layer's final selection, i.e. the
 * selection of its nearest preceding F or R layer, with no rescoring.
 * Every layer then attends over its own selection (SparseAttn).
 *
 * q      : [N][B][Hq][d] bf16 bits;  k[l], v[l]: [B][Hkv][Lmax][d] bf16 bits
 * len    : [B] context lengths (<= Lmax)
 * rho    : pool expansion factor (mode 3 only; >= 1)
 * qbits  : 0, or 2 (mode 3 only): the scores of Eq. (9) use the keys
 *          quantized by Eq. (7)-(8) (prism_ref_quantize_row, groups of
 *          PRISM_REF_QGROUP), dequantized; attention keeps the bf16 keys
 * out    : [N][B][Hq][d] fp64;       idx_out: [N][B][Hkv][kappa] int32
 * pool_out (nullable, mode 3): [N][B][Hkv][rho*kappa] int32, the pool in
 *          effect at each layer (an anchor's own pool, a refined layer's
 *          inherited pool), ascending positions, -1 padded.
 * Query head j uses KV head j / (Hq / Hkv).
 * Returns 0, or -1 on an invalid argument (checked before any work).
 */
int prism_ref_decode_step(int B, int Hq, int Hkv, int d, int Lmax, int kappa,
                          int r, int n_layers, const uint8_t *anchor_mask,
                          int mode, int chain, double scale, int rho, int qbits,
                          const uint16_t *q, const uint16_t *const *k,
                          const uint16_t *const *v, const int32_t *len,
                          double *out, int32_t *idx_out, int32_t *pool_out)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || d < 1 || Lmax < 1 ||
        kappa < 1 || r < 0 || n_layers < 1 || mode < 0 || mode > 3 ||
        chain < 0 || chain > 1)
        return -1;
    if (mode == 3 && (rho < 1 || (long long)rho * kappa > 0x7fffffffLL)) return -1;
    if (qbits != 0 && (qbits != 2 || mode != 3 || d % PRISM_REF_QGROUP != 0)) return -1;
    if (mode != 2) {
        if (anchor_mask[0] != 1) return -1;
        for (int l = 0; l < n_layers; ++l)
            if (anchor_mask[l] > 2) return -1;
    }
    for (int b = 0; b < B; ++b)
        if (len[b] < 0 || len[b] > Lmax) return -1;

    const int G = Hq / Hkv;
    const int rows = B * Hkv;
    const size_t row_sel = (size_t)kappa;
    int last_anchor = 0;
    /* mode 3: the most recent anchor's pool, [rows][n_pool] */
#if PRISM_REF_PLANT == 13
    const int n_pool = kappa;                  /* planted: pool of kappa, not rho*kappa */
#else
    const int n_pool = (mode == 3) ? rho * kappa : 0;
#endif
    int32_t *pool = NULL;
    if (mode == 3) {
        pool = (int32_t *)malloc(sizeof(int32_t) * (size_t)rows * (size_t)n_pool);
        if (!pool) return -1;
    }

    for (int l = 0; l < n_layers; ++l) {
        const int is_anchor = (mode == 2) || anchor_mask[l] == 1;
        const int is_shared = (mode != 2) && anchor_mask[l] == 2;
        int src_layer = l - 1;
#if PRISM_REF_PLANT == 10
        src_layer = last_anchor;               /* planted: ignores the chain choice */
#else
        if (chain == 1) src_layer = last_anchor;
#endif
        int32_t *sel_l = idx_out + (size_t)l * (size_t)rows * row_sel;
        const int32_t *sel_src = (l > 0) ? idx_out + (size_t)src_layer * (size_t)rows * row_sel : NULL;
        /* the previous layer's final selection (what a shared layer keeps) */
#if PRISM_REF_PLANT == 16
        const int32_t *sel_prev = (l > 0) ? idx_out + (size_t)last_anchor * (size_t)rows * row_sel : NULL;   /* planted: the anchor's */
#else
        const int32_t *sel_prev = (l > 0) ? idx_out + (size_t)(l - 1) * (size_t)rows * row_sel : NULL;
#endif

#pragma omp parallel for schedule(dynamic, 1)
        for (int row = 0; row < rows; ++row) {
            const int b = row / Hkv, h = row % Hkv;
            const int L = len[b];
            const uint16_t *qg = q + (((size_t)l * B + b) * Hq + (size_t)h * G) * (size_t)d;
            const uint16_t *kr = k[l] + ((size_t)b * Hkv + h) * (size_t)Lmax * (size_t)d;
            const uint16_t *vr = v[l] + ((size_t)b * Hkv + h) * (size_t)Lmax * (size_t)d;
            int32_t *sel = sel_l + (size_t)row * row_sel;

            if (is_shared) {
                memcpy(sel, sel_prev + (size_t)row * row_sel, sizeof(int32_t) * row_sel);
                if (mode == 3 && pool_out) {
                    int32_t *po = pool_out + ((size_t)l * rows + row) * (size_t)rho * (size_t)kappa;
                    const int32_t *C = pool + (size_t)row * (size_t)n_pool;
                    for (long e = 0; e < (long)rho * kappa; ++e) po[e] = e < n_pool ? C[e] : -1;
                }
            } else if (mode == 3) {
                int32_t *C = pool + (size_t)row * (size_t)n_pool;
                /* qbits == 2: this layer's keys quantized by Eq. (7)-(8); the
                   scores of Eq. (9) use them (Algorithm 1: INT2 keys at the
                   proposal layer and in the refinement) */
                uint8_t *qc = NULL;
                float *qa = NULL, *qb = NULL;
                if (qbits == 2) {
                    const int M = d / PRISM_REF_QGROUP;
                    const size_t nrow = (size_t)(L > 0 ? L : 1);
                    qc = (uint8_t *)malloc(nrow * (size_t)d);
                    qa = (float *)malloc(nrow * (size_t)M * sizeof(float));
                    qb = (float *)malloc(nrow * (size_t)M * sizeof(float));
                    for (int i = 0; i < L; ++i)
                        prism_ref_quantize_row(d, PRISM_REF_QGROUP, kr + (size_t)i * d,
                                               qc + (size_t)i * d, qa + (size_t)i * M,
                                               qb + (size_t)i * M);
                }
#define POOL_SCORE(n_, pos_, s_)                                                          \
    do {                                                                                  \
        if (qbits == 2)                                                                   \
            prism_ref_score_max_q2(d, PRISM_REF_QGROUP, G, qg, qc, qa, qb, (n_), (pos_),  \
                                   scale, (s_));                                          \
        else                                                                              \
            prism_ref_score_max(d, G, qg, kr, (n_), (pos_), scale, (s_));                 \
    } while (0)
                if (is_anchor) {
                    /* Eq. (9) over the whole cache, then the pool of Eq. (4) */
                    double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
                    POOL_SCORE(L, NULL, s);
                    int nc = prism_ref_topk(L, s, NULL, n_pool, C);
                    /* the first kappa of C in score order: the top-kappa of
                       the pool's own scores */
                    double *sc = (double *)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
                    for (int e = 0; e < nc; ++e) sc[e] = s[C[e]];
#if PRISM_REF_PLANT == 15
                    /* planted: the first kappa pool entries in position order */
                    for (int e = 0; e < nc; ++e) sc[e] = -(double)C[e];
#endif
                    prism_ref_topk(nc, sc, C, kappa, sel);
                    free(sc);
                    free(s);
                } else {
                    /* Eq. (5) on the inherited pool, then Eq. (6) */
                    const int32_t *cand = C;
                    int nc = 0;
#if PRISM_REF_PLANT == 14
                    /* planted: rescoring the previous layer's selection */
                    cand = sel_src + (size_t)row * row_sel;
                    while (nc < kappa && cand[nc] >= 0) ++nc;
#else
                    while (nc < n_pool && C[nc] >= 0) ++nc;
#endif
                    double *s = (double *)malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
                    POOL_SCORE(nc, cand, s);
                    prism_ref_topk(nc, s, cand, kappa, sel);
                    free(s);
                }
#undef POOL_SCORE
                free(qc);
                free(qa);
                free(qb);
                if (pool_out) {
                    int32_t *po = pool_out + ((size_t)l * rows + row) * (size_t)rho * (size_t)kappa;
                    for (long e = 0; e < (long)rho * kappa; ++e) po[e] = e < n_pool ? C[e] : -1;
                }
            } else if (is_anchor) {
                double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
                prism_ref_score(d, G, qg, kr, L, NULL, scale, s);
                prism_ref_topk(L, s, NULL, kappa, sel);
                free(s);
            } else if (mode == 1) {
                memcpy(sel, sel_src + (size_t)row * row_sel, sizeof(int32_t) * row_sel);
            } else {
                int32_t *P = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
                int np = prism_ref_expand(L, kappa, sel_src + (size_t)row * row_sel, r, P);
                double *s = (double *)malloc(sizeof(double) * (size_t)(np > 0 ? np : 1));
#if PRISM_REF_PLANT == 11
                /* planted: rescoring with the previous layer's keys */
                const uint16_t *kprev = k[l > 0 ? l - 1 : 0] + ((size_t)b * Hkv + h) * (size_t)Lmax * (size_t)d;
                prism_ref_score(d, G, qg, kprev, np, P, scale, s);
#else
                prism_ref_score(d, G, qg, kr, np, P, scale, s);
#endif
                prism_ref_topk(np, s, P, kappa, sel);
                free(s);
                free(P);
            }
            double *o = out + (((size_t)l * B + b) * Hq + (size_t)h * G) * (size_t)d;
            prism_ref_attention(d, G, qg, kr, vr, kappa, sel, scale, o, NULL);
        }
        if (is_anchor) last_anchor = l;
    }
    free(pool);
    return 0;
}
