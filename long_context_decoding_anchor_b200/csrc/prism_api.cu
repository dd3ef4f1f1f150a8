// prism_api.cu -- the C ABI (include/prism.h): host-side validation, the
// workspace layout, and the stream-ordered orchestration of the decode step
// (Algorithm 1 of "Prism Attention").
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>

#include "prism.h"
#include "prism_internal.cuh"

using namespace prism;

namespace {
thread_local uint64_t g_launches = 0;
}  // namespace

void prism::count_launches(int n) { g_launches += (uint64_t)n; }

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
    size_t status, hist, ctl, ctl_end;   // [hist, ctl_end) is zeroed per call
    size_t S, cpos, tie, sel, idx[3], pacc, pml, total;
};

Layout make_layout(const prism_config_t &c) {
    const size_t rows = (size_t)c.batch * c.n_kv_heads;
    const size_t G = (size_t)(c.n_q_heads / c.n_kv_heads);
    const size_t nsplit = ((size_t)c.kappa + kAttnChunk - 1) / kAttnChunk;
    Layout l{};
    size_t off = 0;
    l.status = off; off = align256(off + sizeof(DevStatus));
    l.hist = off;   off = align256(off + rows * kHistBins * sizeof(uint32_t));
    l.ctl = off;    off = align256(off + rows * sizeof(RowCtl));
    l.ctl_end = off;
    l.S = off;      off = align256(off + rows * (size_t)c.max_len * sizeof(float));
    l.cpos = off;   off = align256(off + rows * (size_t)c.max_len * sizeof(int32_t));
    l.tie = off;    off = align256(off + rows * (size_t)c.max_len * sizeof(uint64_t));
    l.sel = off;    off = align256(off + rows * (size_t)c.kappa * sizeof(int32_t));
    for (int i = 0; i < 3; ++i) {
        l.idx[i] = off;
        off = align256(off + rows * (size_t)c.kappa * sizeof(int32_t));
    }
    l.pacc = off;   off = align256(off + rows * nsplit * G * (size_t)c.head_dim * sizeof(float));
    l.pml = off;    off = align256(off + rows * nsplit * G * 2 * sizeof(float));
    l.total = off;
    return l;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

prism_status_t check_config(const prism_config_t *c) {
    if (!c) return PRISM_ERR_INVALID_ARG;
    if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->max_len < 1 || c->kappa < 1 ||
        c->radius < 0)
        return PRISM_ERR_INVALID_ARG;
    if (c->n_q_heads % c->n_kv_heads != 0) return PRISM_ERR_INVALID_ARG;
    if (!(c->scale >= 0.f) || std::isinf(c->scale)) return PRISM_ERR_INVALID_ARG;
    if (c->mode < PRISM_MODE_REFINE || c->mode > PRISM_MODE_DENSE_ANCHOR) return PRISM_ERR_INVALID_ARG;
    if (c->chain < PRISM_CHAIN_PREV || c->chain > PRISM_CHAIN_ANCHOR) return PRISM_ERR_INVALID_ARG;
    if (c->head_dim != 64 && c->head_dim != 128) return PRISM_ERR_UNSUPPORTED;
    const int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return PRISM_ERR_UNSUPPORTED;
    if (G > c->head_dim / 8) return PRISM_ERR_UNSUPPORTED;
    if (c->max_len > PRISM_MAX_LEN || c->kappa > PRISM_MAX_LEN) return PRISM_ERR_UNSUPPORTED;
    if ((long long)c->batch * c->n_kv_heads > PRISM_MAX_BATCH_ROWS) return PRISM_ERR_UNSUPPORTED;
    return PRISM_OK;
}

float eff_scale(const prism_config_t &c) {
    return c.scale > 0.f ? c.scale : 1.0f / std::sqrt((float)c.head_dim);
}

uint64_t wait_limit_ns() {
    static uint64_t v = 0;
    if (v == 0) {
        uint64_t ms = 4000;
        if (const char *e = std::getenv("PRISM_WAIT_LIMIT_MS")) {
            long long x = std::atoll(e);
            if (x > 0) ms = (uint64_t)x;
        }
        v = ms * 1000000ull;
    }
    return v;
}

int num_sms() {
    static int cache[128] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

struct Ws {
    DevStatus *st;
    uint32_t *hist;
    RowCtl *ctl;
    float *S;
    int32_t *cpos;
    uint64_t *tie;
    int32_t *sel;
    int32_t *idx[3];
    float *pacc, *pml;
    uint8_t *base;
    Layout l;
};

prism_status_t carve(const prism_config_t &c, void *ws, size_t ws_bytes, Ws *w) {
    if (!ws || !aligned(ws, 256)) return PRISM_ERR_INVALID_ARG;
    w->l = make_layout(c);
    if (ws_bytes < w->l.total) return PRISM_ERR_WORKSPACE;
    uint8_t *b = static_cast<uint8_t *>(ws);
    w->base = b;
    w->st = reinterpret_cast<DevStatus *>(b + w->l.status);
    w->hist = reinterpret_cast<uint32_t *>(b + w->l.hist);
    w->ctl = reinterpret_cast<RowCtl *>(b + w->l.ctl);
    w->S = reinterpret_cast<float *>(b + w->l.S);
    w->cpos = reinterpret_cast<int32_t *>(b + w->l.cpos);
    w->tie = reinterpret_cast<uint64_t *>(b + w->l.tie);
    w->sel = reinterpret_cast<int32_t *>(b + w->l.sel);
    for (int i = 0; i < 3; ++i) w->idx[i] = reinterpret_cast<int32_t *>(b + w->l.idx[i]);
    w->pacc = reinterpret_cast<float *>(b + w->l.pacc);
    w->pml = reinterpret_cast<float *>(b + w->l.pml);
    return PRISM_OK;
}

prism_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA; }

#define PRISM_TRY(expr)                              \
    do {                                             \
        prism_status_t _s = (expr);                  \
        if (_s != PRISM_OK) return _s;               \
    } while (0)
#define PRISM_CUDA(expr) PRISM_TRY(cuda_status(expr))

prism_status_t zero_control(const Ws &w, cudaStream_t s) {
    return cuda_status(cudaMemsetAsync(w.base + w.l.hist, 0, w.l.ctl_end - w.l.hist, s));
}

// Anchor: Eq. (1) over every token, then Eq. (2).
prism_status_t run_anchor(const prism_config_t &c, const Ws &w, const void *q, const void *k,
                          const int32_t *len, int32_t *idx_out, float *scores, cudaStream_t s) {
    ScoreArgs sa{};
    sa.q = q; sa.k = k; sa.len = len;
    sa.B = c.batch; sa.Hkv = c.n_kv_heads; sa.G = c.n_q_heads / c.n_kv_heads;
    sa.d = c.head_dim; sa.Lmax = c.max_len; sa.scale = eff_scale(c);
    sa.S = scores ? scores : w.S; sa.hist = w.hist; sa.cpos = nullptr; sa.ctl = w.ctl;
    sa.st = w.st; sa.wait_ns = wait_limit_ns();
    PRISM_CUDA(launch_anchor_score(sa, num_sms(), s));
    SelectArgs se{};
    se.S = sa.S; se.cpos = nullptr; se.len = len;
    se.B = c.batch; se.Hkv = c.n_kv_heads; se.Lmax = c.max_len; se.kappa = c.kappa;
    se.hist = w.hist; se.ctl = w.ctl; se.sel = w.sel; se.tie = w.tie; se.idx_out = idx_out;
    se.st = w.st;
    PRISM_CUDA(launch_select(se, c.max_len, s));
    return PRISM_OK;
}

long long proposal_bound(const prism_config_t &c) {
    const long long win = 2LL * c.radius + 1;
    const long long b = (long long)c.kappa * win;
    return b < c.max_len ? b : c.max_len;
}

// Refined layer: +-r proposal, Eq. (5) on it, Eq. (6).
prism_status_t run_refine(const prism_config_t &c, const Ws &w, const void *q, const void *k,
                          const int32_t *len, const int32_t *idx_prev, int32_t *idx_out,
                          cudaStream_t s) {
    ExpandArgs ea{};
    ea.idx_prev = idx_prev; ea.len = len; ea.B = c.batch; ea.Hkv = c.n_kv_heads;
    ea.Lmax = c.max_len; ea.kappa = c.kappa; ea.radius = c.radius;
    ea.cpos = w.cpos; ea.ctl = w.ctl; ea.st = w.st;
    PRISM_CUDA(launch_expand(ea, s));
    ScoreArgs sa{};
    sa.q = q; sa.k = k; sa.len = len;
    sa.B = c.batch; sa.Hkv = c.n_kv_heads; sa.G = c.n_q_heads / c.n_kv_heads;
    sa.d = c.head_dim; sa.Lmax = c.max_len; sa.scale = eff_scale(c);
    sa.S = w.S; sa.hist = w.hist; sa.cpos = w.cpos; sa.ctl = w.ctl;
    sa.st = w.st; sa.wait_ns = wait_limit_ns();
    const long long bound = proposal_bound(c);
    PRISM_CUDA(launch_refine_rescore(sa, bound, s));
    SelectArgs se{};
    se.S = w.S; se.cpos = w.cpos; se.len = len;
    se.B = c.batch; se.Hkv = c.n_kv_heads; se.Lmax = c.max_len; se.kappa = c.kappa;
    se.hist = w.hist; se.ctl = w.ctl; se.sel = w.sel; se.tie = w.tie; se.idx_out = idx_out;
    se.st = w.st;
    PRISM_CUDA(launch_select(se, bound, s));
    return PRISM_OK;
}

prism_status_t run_attn(const prism_config_t &c, const Ws &w, const void *q, const void *k,
                        const void *v, const int32_t *len, const int32_t *idx, int idx_stride,
                        int n_idx, void *out, cudaStream_t s) {
    AttnArgs aa{};
    aa.q = q; aa.k = k; aa.v = v; aa.len = len; aa.idx = idx;
    aa.idx_stride = idx_stride; aa.n_idx = n_idx;
    aa.B = c.batch; aa.Hkv = c.n_kv_heads; aa.G = c.n_q_heads / c.n_kv_heads;
    aa.d = c.head_dim; aa.Lmax = c.max_len; aa.scale = eff_scale(c);
    aa.part_acc = w.pacc; aa.part_ml = w.pml; aa.out = out; aa.st = w.st;
    PRISM_CUDA(launch_sparse_attn(aa, s));
    return PRISM_OK;
}

}  // namespace

extern "C" {

prism_status_t prism_workspace_size(const prism_config_t *cfg, size_t *bytes) {
    PRISM_TRY(check_config(cfg));
    if (!bytes) return PRISM_ERR_INVALID_ARG;
    *bytes = make_layout(*cfg).total;
    return PRISM_OK;
}

prism_status_t prism_index_anchor(const prism_config_t *cfg, const void *q, const void *k,
                                  const int32_t *len, int32_t *idx_out, float *scores_out,
                                  void *ws, size_t ws_bytes, void *stream) {
    PRISM_TRY(check_config(cfg));
    if (!q || !k || !len || !idx_out) return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(len, 4) || !aligned(idx_out, 4) ||
        (scores_out && !aligned(scores_out, 4)))
        return PRISM_ERR_INVALID_ARG;
    Ws w;
    PRISM_TRY(carve(*cfg, ws, ws_bytes, &w));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PRISM_TRY(zero_control(w, s));
    return run_anchor(*cfg, w, q, k, len, idx_out, scores_out, s);
}

prism_status_t prism_score_anchor(const prism_config_t *cfg, const void *q, const void *k,
                                  const int32_t *len, float *scores_out, void *ws,
                                  size_t ws_bytes, void *stream) {
    PRISM_TRY(check_config(cfg));
    if (!q || !k || !len || !scores_out) return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(len, 4) || !aligned(scores_out, 4))
        return PRISM_ERR_INVALID_ARG;
    Ws w;
    PRISM_TRY(carve(*cfg, ws, ws_bytes, &w));
    const prism_config_t &c = *cfg;
    ScoreArgs sa{};
    sa.q = q; sa.k = k; sa.len = len;
    sa.B = c.batch; sa.Hkv = c.n_kv_heads; sa.G = c.n_q_heads / c.n_kv_heads;
    sa.d = c.head_dim; sa.Lmax = c.max_len; sa.scale = eff_scale(c);
    sa.S = scores_out; sa.hist = w.hist; sa.cpos = nullptr; sa.ctl = w.ctl;
    sa.st = w.st; sa.wait_ns = wait_limit_ns();
    return cuda_status(launch_anchor_score(sa, num_sms(), static_cast<cudaStream_t>(stream)));
}

prism_status_t prism_index_refine(const prism_config_t *cfg, const void *q, const void *k,
                                  const int32_t *len, const int32_t *idx_prev, int32_t *idx_out,
                                  int32_t *cand_pos, float *cand_score, int32_t *cand_count,
                                  int32_t cand_cap, void *ws, size_t ws_bytes, void *stream) {
    PRISM_TRY(check_config(cfg));
    if (!q || !k || !len || !idx_prev || !idx_out || idx_prev == idx_out)
        return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(len, 4) || !aligned(idx_prev, 4) ||
        !aligned(idx_out, 4))
        return PRISM_ERR_INVALID_ARG;
    const bool any = cand_pos || cand_score || cand_count;
    const bool all = cand_pos && cand_score && cand_count;
    if (any && (!all || cand_cap < 1 || !aligned(cand_pos, 4) || !aligned(cand_score, 4) ||
                !aligned(cand_count, 4)))
        return PRISM_ERR_INVALID_ARG;
    Ws w;
    PRISM_TRY(carve(*cfg, ws, ws_bytes, &w));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PRISM_TRY(zero_control(w, s));
    PRISM_TRY(run_refine(*cfg, w, q, k, len, idx_prev, idx_out, s));
    if (all)
        PRISM_CUDA(launch_export_candidates(w.S, w.cpos, w.ctl, cfg->batch * cfg->n_kv_heads,
                                            cfg->max_len, cand_pos, cand_score, cand_count,
                                            cand_cap, s));
    return PRISM_OK;
}

prism_status_t prism_sparse_decode(const prism_config_t *cfg, const void *q, const void *k,
                                   const void *v, const int32_t *len, const int32_t *idx,
                                   int32_t n_idx, void *out, void *ws, size_t ws_bytes,
                                   void *stream) {
    PRISM_TRY(check_config(cfg));
    if (!q || !k || !v || !len || !idx || !out) return PRISM_ERR_INVALID_ARG;
    if (n_idx < 1 || n_idx > cfg->kappa) return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(len, 4) || !aligned(idx, 4))
        return PRISM_ERR_INVALID_ARG;
    Ws w;
    PRISM_TRY(carve(*cfg, ws, ws_bytes, &w));
    return run_attn(*cfg, w, q, k, v, len, idx, n_idx, n_idx, out,
                    static_cast<cudaStream_t>(stream));
}

prism_status_t prism_decode_step(const prism_config_t *cfg, const void *q, const void *const *k,
                                 const void *const *v, const int32_t *len, void *out,
                                 int32_t *idx_out, void *ws, size_t ws_bytes, void *stream) {
    PRISM_TRY(check_config(cfg));
    const prism_config_t &c = *cfg;
    if (c.n_layers < 1 || !q || !k || !v || !len || !out) return PRISM_ERR_INVALID_ARG;
    if (c.mode != PRISM_MODE_DENSE_ANCHOR) {
        if (!c.anchor_mask || !c.anchor_mask[0]) return PRISM_ERR_INVALID_ARG;
    }
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(len, 4) ||
        (idx_out && !aligned(idx_out, 4)))
        return PRISM_ERR_INVALID_ARG;
    for (int l = 0; l < c.n_layers; ++l) {
        if (!k[l] || !v[l] || !aligned(k[l], 16) || !aligned(v[l], 16)) return PRISM_ERR_INVALID_ARG;
    }
    Ws w;
    PRISM_TRY(carve(c, ws, ws_bytes, &w));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PRISM_TRY(zero_control(w, s));

    const size_t rows = (size_t)c.batch * c.n_kv_heads;
    const size_t sel_elems = rows * (size_t)c.kappa;
    const size_t q_elems = (size_t)c.batch * c.n_q_heads * c.head_dim;
    const uint16_t *qb = static_cast<const uint16_t *>(q);
    uint16_t *ob = static_cast<uint16_t *>(out);

    const int32_t *anchor_sel = nullptr;   // most recent anchor layer's selection
    const int32_t *prev_sel = nullptr;     // previous layer's selection
    int flip = 0;
    for (int l = 0; l < c.n_layers; ++l) {
        const bool anchor = c.mode == PRISM_MODE_DENSE_ANCHOR || c.anchor_mask[l];
        const void *ql = qb + (size_t)l * q_elems;
        const int32_t *src = c.chain == PRISM_CHAIN_ANCHOR ? anchor_sel : prev_sel;
        const int32_t *cur = nullptr;
        if (anchor) {
            int32_t *dst = idx_out ? idx_out + (size_t)l * sel_elems : w.idx[2];
            PRISM_TRY(run_anchor(c, w, ql, k[l], len, dst, nullptr, s));
            cur = dst;
            anchor_sel = dst;
        } else if (c.mode == PRISM_MODE_STATIC_REUSE) {
            if (idx_out) {
                int32_t *dst = idx_out + (size_t)l * sel_elems;
                PRISM_CUDA(cudaMemcpyAsync(dst, src, sel_elems * sizeof(int32_t),
                                           cudaMemcpyDeviceToDevice, s));
                cur = dst;
            } else {
                cur = src;
            }
        } else {
            int32_t *dst = idx_out ? idx_out + (size_t)l * sel_elems : w.idx[flip];
            flip ^= 1;
            PRISM_TRY(run_refine(c, w, ql, k[l], len, src, dst, s));
            cur = dst;
        }
        PRISM_TRY(run_attn(c, w, ql, k[l], v[l], len, cur, c.kappa, c.kappa,
                           ob + (size_t)l * q_elems, s));
        prev_sel = cur;
    }
    return PRISM_OK;
}

prism_status_t prism_check_device_status(void *ws, size_t ws_bytes, void *stream,
                                         uint32_t detail[4]) {
    if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(DevStatus)) return PRISM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DevStatus h{};
    PRISM_CUDA(cudaMemcpyAsync(&h, ws, sizeof(DevStatus), cudaMemcpyDeviceToHost, s));
    PRISM_CUDA(cudaStreamSynchronize(s));
    if (detail) {
        detail[0] = h.code;
        detail[1] = h.where;
        detail[2] = h.value;
        detail[3] = 0;
    }
    if (h.code != kDevErrNone) {
        PRISM_CUDA(cudaMemsetAsync(ws, 0, sizeof(DevStatus), s));
        PRISM_CUDA(cudaStreamSynchronize(s));
    }
    if (h.code == kDevErrNone) return PRISM_OK;
    if (h.code == kDevErrTimeout) return PRISM_ERR_TIMEOUT;
    return PRISM_ERR_DEVICE;
}

prism_status_t prism_debug_wait_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns,
                                        void *stream) {
    if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(DevStatus)) return PRISM_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 10ull * 1000000000ull) return PRISM_ERR_INVALID_ARG;
    return cuda_status(launch_debug_wait(static_cast<DevStatus *>(ws), limit_ns,
                                         static_cast<cudaStream_t>(stream)));
}

const char *prism_status_string(prism_status_t st) {
    switch (st) {
        case PRISM_OK: return "ok";
        case PRISM_ERR_INVALID_ARG: return "invalid argument";
        case PRISM_ERR_UNSUPPORTED: return "unsupported shape";
        case PRISM_ERR_WORKSPACE: return "workspace too small";
        case PRISM_ERR_CUDA: return "CUDA launch or runtime error";
        case PRISM_ERR_TIMEOUT: return "a bounded device wait timed out";
        case PRISM_ERR_DEVICE: return "device-side contract violation";
    }
    return "unknown status";
}

uint64_t prism_launch_count(void) { return g_launches; }

int32_t prism_version(void) { return 100; }

}  // extern "C"
