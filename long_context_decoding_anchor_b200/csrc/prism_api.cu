// prism_api.cu -- the C ABI (include/prism.h): host-side validation, the
// workspace layout, and the orchestration of the decode step (Algorithm 1 of
// "Prism Attention").
//
// The decode step is a DAG, not a chain.  An anchor layer's scoring reads only
// its own inputs, so it can run ahead of the refined layers; a layer's
// attention reads only its own selection, so it can trail behind.  The step
// therefore runs on three streams forked from the caller's stream and joined
// back into it (events, so a CUDA-graph capture records the same DAG):
//   A (low priority):  each anchor layer's scoring and top-kappa, at most two
//                      anchors ahead of the chain (two workspace slots);
//   M (high priority): the refined layers in order -- rescoring, top-kappa --
//                      each anchor's group waiting for that anchor's selection;
//   C (high priority): each layer's sparse attention once its selection is
//                      done.
// In pool mode a fourth stream X (high priority) selects each anchor's pool
// and its own top-kappa while A scans the next anchor, and the refined layers
// of each group rescore their anchor's pool together (one launch of each
// kernel per group) once the pool is selected.
// PRISM_FLAG_SERIAL runs everything on the caller's stream instead.
//
// The context-parallel calls (include/prism_cp.h, at the end of this file)
// run the same kernels on one rank's shard of the positions, with the
// helpers of cp.cu around them.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "cp_internal.cuh"
#include "prism.h"
#include "prism_cp.h"
#include "prism_internal.cuh"

using namespace prism;

namespace {
thread_local uint64_t g_launches = 0;
}  // namespace

void prism::count_launches(int n) { g_launches += (uint64_t)n; }

bool prism::use_pdl() {
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("PRISM_NO_PDL");
        v = (e && e[0] == '1') ? 0 : 1;
    }
    return v == 1;
}

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kAnchorAhead = 2;     // anchors indexed ahead of the chain (ring of anchor slots)

// Buffers of one anchor selection slot.
struct SlotLayout {
    size_t hist, S, cspill;
};

// The rescoring of a refined layer with source entries E and radius r, in
// launches of up to nzmax batched layers: runs per row (the largest P * K of
// refine_parts over the batch sizes) and the ties' overflow capacity.
struct RunLayout {
    int E, radius, nzmax, nruns, tie_cap;
    int parts1;                     // parts of a single-layer launch (the fused selection)
};

struct Layout {
    size_t status;
    size_t ctl_begin, ctl_end;      // [ctl_begin, ctl_end): histograms and counters; zeroed per call
    SlotLayout slot[kAnchorAhead];
    size_t attn_ctl;
    RunLayout rl;
    size_t rhist, runs, run_cnt, ties;   // [nzmax][rows][...] candidate runs of refined layers
    size_t rbar, part_cnt;               // fused selection: arrivals [rows], counts [rows][parts1][2]
    size_t canon, idx_all, pool_all, pacc, pml, total;
};

int n_layers_of(const prism_config_t &c) { return c.n_layers > 0 ? c.n_layers : 1; }

bool pool_mode(const prism_config_t &c) { return c.mode == PRISM_MODE_POOL; }

// Entries of the selection a refined layer starts from: the anchor's pool of
// rho * kappa tokens in pool mode, a selection of kappa tokens otherwise.
int src_kappa_of(const prism_config_t &c) {
    return pool_mode(c) ? c.pool_factor * c.kappa : c.kappa;
}

// Radius of a refined layer's proposal: the pool is rescored as it is.
int refine_radius_of(const prism_config_t &c) { return pool_mode(c) ? 0 : c.radius; }

RunLayout run_layout(const prism_config_t &c, int E, int radius, int nzmax) {
    const int rows = c.batch * c.n_kv_heads;
    RunLayout r{E, radius, nzmax, 1, 1, refine_parts(E, radius, c.max_len, rows, 1).parts};
    for (int nz = 1; nz <= nzmax; ++nz) {
        const RefineParts rp = refine_parts(E, radius, c.max_len, rows, nz);
        r.nruns = std::max(r.nruns, rp.parts * rp.run_k);
    }
    r.tie_cap = (int)std::min<long long>(c.max_len, (long long)r.nruns * kRunCap);
    return r;
}

// The layout of a workspace.  A context-parallel rank passes its shard's
// refined-layer source (E entries, radius 0) instead of the config's.
Layout make_layout(const prism_config_t &c, int src_E = -1, int src_r = -1) {
    const size_t rows = (size_t)c.batch * c.n_kv_heads;
    const size_t G = (size_t)(c.n_q_heads / c.n_kv_heads);
    const size_t nsplit = ((size_t)c.kappa + kAttnChunk - 1) / kAttnChunk;
    const size_t sel_elems = rows * (size_t)c.kappa;
    const size_t src_elems = rows * (size_t)src_kappa_of(c);
    const size_t n_pools = pool_mode(c) ? (size_t)n_layers_of(c) : 0;
    Layout l{};
    l.rl = run_layout(c, src_E >= 0 ? src_E : src_kappa_of(c), src_r >= 0 ? src_r : refine_radius_of(c),
                      pool_mode(c) ? kMaxZ : 1);
    const size_t nzs = (size_t)l.rl.nzmax;
    size_t off = 0;
    l.status = off; off = align256(off + sizeof(DevStatus));
    l.ctl_begin = off;
    for (int s = 0; s < kAnchorAhead; ++s) {
        l.slot[s].hist = off;   off = align256(off + rows * kHistBins * sizeof(uint32_t));
    }
    l.attn_ctl = off; off = align256(off + rows * sizeof(RowCtl));
    l.rhist = off;    off = align256(off + nzs * rows * kHistBins * sizeof(uint32_t));
    l.rbar = off;     off = align256(off + rows * sizeof(uint32_t));
    l.ctl_end = off;
    l.part_cnt = off; off = align256(off + rows * (size_t)l.rl.parts1 * 2 * sizeof(int32_t));
    l.runs = off;     off = align256(off + nzs * rows * (size_t)l.rl.nruns * kRunCap * sizeof(uint64_t));
    l.run_cnt = off;  off = align256(off + nzs * rows * (size_t)l.rl.nruns * sizeof(int32_t));
    l.ties = off;     off = align256(off + nzs * rows * (size_t)l.rl.tie_cap * sizeof(uint64_t));
    for (int s = 0; s < kAnchorAhead; ++s) {
        l.slot[s].S = off;      off = align256(off + rows * (size_t)c.max_len * sizeof(float));
        l.slot[s].cspill = off; off = align256(off + rows * 2 * (size_t)c.max_len * sizeof(uint64_t));
    }
    l.canon = off;     off = align256(off + src_elems * sizeof(int32_t));
    l.idx_all = off;   off = align256(off + (size_t)n_layers_of(c) * sel_elems * sizeof(int32_t));
    l.pool_all = off;  off = align256(off + n_pools * src_elems * sizeof(int32_t));
    l.pacc = off;      off = align256(off + rows * nsplit * G * (size_t)c.head_dim * sizeof(float));
    l.pml = off;       off = align256(off + rows * nsplit * G * 2 * sizeof(float));
    l.total = off;
    return l;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

prism_status_t check_config(const prism_config_t *c) {
    if (!c) return PRISM_ERR_INVALID_ARG;
    if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->max_len < 1 || c->kappa < 1 ||
        c->radius < 0 || c->n_layers < 0)
        return PRISM_ERR_INVALID_ARG;
    if (c->n_q_heads % c->n_kv_heads != 0) return PRISM_ERR_INVALID_ARG;
    if (!(c->scale >= 0.f) || std::isinf(c->scale)) return PRISM_ERR_INVALID_ARG;
    if (c->mode < PRISM_MODE_REFINE || c->mode > PRISM_MODE_POOL) return PRISM_ERR_INVALID_ARG;
    if (c->mode == PRISM_MODE_POOL && c->pool_factor < 1) return PRISM_ERR_INVALID_ARG;
    if (c->chain < PRISM_CHAIN_PREV || c->chain > PRISM_CHAIN_ANCHOR) return PRISM_ERR_INVALID_ARG;
    if (c->flags & ~(PRISM_FLAG_SERIAL | PRISM_FLAG_INT2_KEYS)) return PRISM_ERR_INVALID_ARG;
    // 2-bit proposal keys belong to the pool mode (Eq. (9) scores)
    if ((c->flags & PRISM_FLAG_INT2_KEYS) && c->mode != PRISM_MODE_POOL) return PRISM_ERR_INVALID_ARG;
    if (c->head_dim != 64 && c->head_dim != 128) return PRISM_ERR_UNSUPPORTED;
    const int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return PRISM_ERR_UNSUPPORTED;
    if (G > c->head_dim / 8) return PRISM_ERR_UNSUPPORTED;
    if (c->max_len > PRISM_MAX_LEN || c->kappa > PRISM_MAX_LEN) return PRISM_ERR_UNSUPPORTED;
    if (c->mode == PRISM_MODE_POOL && (long long)c->pool_factor * c->kappa > PRISM_MAX_LEN)
        return PRISM_ERR_UNSUPPORTED;
    if ((long long)c->batch * c->n_kv_heads > PRISM_MAX_BATCH_ROWS) return PRISM_ERR_UNSUPPORTED;
    if (c->n_layers > PRISM_MAX_LAYERS) return PRISM_ERR_UNSUPPORTED;
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

constexpr int kMaxDevices = 64;

int num_sms() {
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Helper streams and a pool of events, per device, created on first use and
// kept until the process exits.
struct DeviceHelpers {
    cudaStream_t anchor = nullptr, chain = nullptr, attn = nullptr;
    cudaStream_t aux = nullptr;     // pool mode: the anchors' two selections
    std::vector<cudaEvent_t> events;
};
std::mutex g_helpers_mu;
DeviceHelpers g_helpers[kMaxDevices];

prism_status_t helpers_for_current_device(size_t n_events, DeviceHelpers **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PRISM_ERR_CUDA;
    DeviceHelpers &h = g_helpers[dev];
    if (!h.anchor) {
        int lo = 0, hi = 0;
        if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return PRISM_ERR_CUDA;
        // lo is the least urgent priority, hi the most urgent.
        if (cudaStreamCreateWithPriority(&h.anchor, cudaStreamNonBlocking, lo) != cudaSuccess ||
            cudaStreamCreateWithPriority(&h.chain, cudaStreamNonBlocking, hi) != cudaSuccess ||
            cudaStreamCreateWithPriority(&h.attn, cudaStreamNonBlocking, hi) != cudaSuccess ||
            cudaStreamCreateWithPriority(&h.aux, cudaStreamNonBlocking, hi) != cudaSuccess)
            return PRISM_ERR_CUDA;
    }
    while (h.events.size() < n_events) {
        cudaEvent_t e;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return PRISM_ERR_CUDA;
        h.events.push_back(e);
    }
    *out = &h;
    return PRISM_OK;
}

struct Slot {
    uint32_t *hist;
    float *S;
    uint64_t *cspill;
};

struct Ws {
    DevStatus *st;
    Slot slot[kAnchorAhead];
    RowCtl *attn_ctl;
    uint32_t *rhist;                      // [nzmax][rows][kHistBins]
    uint64_t *runs;                       // [nzmax][rows][nruns][kRunCap]
    int32_t *run_cnt;                     // [nzmax][rows][nruns]
    uint64_t *ties;                       // [nzmax][rows][tie_cap]
    uint32_t *rbar;                       // fused selection: arrival counters [rows]
    int32_t *part_cnt;                    // fused selection: [rows][parts][2]
    mutable uint32_t bar_arrivals = 0;    // arrivals enqueued so far in this call (host side)
    int32_t *canon;
    int32_t *idx_all;
    int32_t *pool_all;                    // pool mode: [N][rows][rho*kappa]
    float *pacc, *pml;
    uint8_t *base;
    Layout l;
};

prism_status_t carve(const prism_config_t &c, void *ws, size_t ws_bytes, Ws *w, int src_E = -1,
                     int src_r = -1) {
    if (!ws || !aligned(ws, 256)) return PRISM_ERR_INVALID_ARG;
    w->l = make_layout(c, src_E, src_r);
    if (ws_bytes < w->l.total) return PRISM_ERR_WORKSPACE;
    uint8_t *b = static_cast<uint8_t *>(ws);
    w->base = b;
    w->st = reinterpret_cast<DevStatus *>(b + w->l.status);
    for (int s = 0; s < kAnchorAhead; ++s) {
        w->slot[s].hist = reinterpret_cast<uint32_t *>(b + w->l.slot[s].hist);
        w->slot[s].S = reinterpret_cast<float *>(b + w->l.slot[s].S);
        w->slot[s].cspill = reinterpret_cast<uint64_t *>(b + w->l.slot[s].cspill);
    }
    w->attn_ctl = reinterpret_cast<RowCtl *>(b + w->l.attn_ctl);
    w->rhist = reinterpret_cast<uint32_t *>(b + w->l.rhist);
    w->runs = reinterpret_cast<uint64_t *>(b + w->l.runs);
    w->run_cnt = reinterpret_cast<int32_t *>(b + w->l.run_cnt);
    w->ties = reinterpret_cast<uint64_t *>(b + w->l.ties);
    w->rbar = reinterpret_cast<uint32_t *>(b + w->l.rbar);
    w->part_cnt = reinterpret_cast<int32_t *>(b + w->l.part_cnt);
    w->bar_arrivals = 0;
    w->canon = reinterpret_cast<int32_t *>(b + w->l.canon);
    w->idx_all = reinterpret_cast<int32_t *>(b + w->l.idx_all);
    w->pool_all = reinterpret_cast<int32_t *>(b + w->l.pool_all);
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
    return cuda_status(cudaMemsetAsync(w.base + w.l.ctl_begin, 0, w.l.ctl_end - w.l.ctl_begin, s));
}

ScoreArgs score_args(const prism_config_t &c, const Ws &w, const void *q, const void *k,
                     const int32_t *len) {
    ScoreArgs sa{};
    sa.q = q; sa.k = k; sa.len = len;
    sa.B = c.batch; sa.Hkv = c.n_kv_heads; sa.G = c.n_q_heads / c.n_kv_heads;
    sa.d = c.head_dim; sa.Lmax = c.max_len; sa.scale = eff_scale(c);
    sa.kappa = c.kappa; sa.radius = c.radius; sa.st = w.st; sa.wait_ns = wait_limit_ns();
    sa.agg = pool_mode(c) ? kAggMax : kAggSum;
    sa.q2 = (c.flags & PRISM_FLAG_INT2_KEYS) ? 1 : 0;
    return sa;
}

SelectArgs select_args(const prism_config_t &c, const Ws &w, const Slot &sl, const int32_t *len,
                       int32_t *idx_out) {
    SelectArgs se{};
    se.S = sl.S; se.len = len;
    se.B = c.batch; se.Hkv = c.n_kv_heads; se.Lmax = c.max_len; se.kappa = c.kappa;
    se.radius = c.radius;
    se.hist = sl.hist; se.cspill = sl.cspill;
    se.idx_out = idx_out; se.st = w.st; se.wait_ns = wait_limit_ns();
    return se;
}

// Anchor scoring (Eq. (1)) into slot `slot`; scores go to `scores` if given.
prism_status_t run_anchor_score(const prism_config_t &c, const Ws &w, int slot, const void *q,
                                const void *k, const int32_t *len, float *scores,
                                cudaStream_t s) {
    ScoreArgs sa = score_args(c, w, q, k, len);
    sa.S = scores ? scores : w.slot[slot].S;
    sa.hist = w.slot[slot].hist;
    return cuda_status(launch_anchor_score(sa, num_sms(), s));
}

// Anchor top-kappa (Eq. (2)) from slot `slot`.
prism_status_t run_anchor_select(const prism_config_t &c, const Ws &w, int slot,
                                 const int32_t *len, int32_t *idx_out, cudaStream_t s) {
    return cuda_status(launch_select(select_args(c, w, w.slot[slot], len, idx_out), s));
}

// Pool mode, proposal layer: from the scores and histogram in slot `slot`,
// the pool of Eq. (4) (rho * kappa tokens) and the layer's own top-kappa.
// The first selection leaves the histogram for the second, which clears it.
prism_status_t run_pool_select(const prism_config_t &c, const Ws &w, int slot, const int32_t *len,
                               int32_t *pool_out, int32_t *idx_out, cudaStream_t s) {
    SelectArgs p = select_args(c, w, w.slot[slot], len, pool_out);
    p.kappa = src_kappa_of(c);
    p.radius = 0;
    p.keep_hist = 1;
    PRISM_CUDA(launch_select(p, s));
    return cuda_status(launch_select(select_args(c, w, w.slot[slot], len, idx_out), s));
}

// Refined layers: Eq. (5) over the proposal of the canonical source `src` (E
// entries, radius r) with each of nz layers' own q and K, then Eq. (6): one
// launch of each kernel for all of them (layer z in grid z).  Layer z's
// selection goes to outs[z].  Spos (nullable, nz == 1) receives every
// candidate's score by position (row stride spos_stride).  `alone` says that
// no other kernel of the call can run beside this one (no anchor scan in
// flight); it decides how a layer selects in place (below).
// A context-parallel rank's refined layer: the source is global, len is the
// shard's, and the proposal is cut to [lo, lo + len) (see ScoreArgs::glen).
struct CutToShard {
    const int32_t *glen;
    int glmax, lo;
};

prism_status_t run_refine_batch(const prism_config_t &c, const Ws &w, const void *const *qs,
                                const void *const *ks, int32_t *const *outs, int nz,
                                const int32_t *len, const int32_t *src, int E, int radius,
                                float *Spos, int spos_stride, cudaStream_t s, bool alone = true,
                                const CutToShard *cut = nullptr) {
    if (nz < 1 || nz > w.l.rl.nzmax || E != w.l.rl.E || radius != w.l.rl.radius)
        return PRISM_ERR_INVALID_ARG;
    const size_t rows = (size_t)c.batch * c.n_kv_heads;
    const RefineParts rp = refine_parts(E, radius, c.max_len, (int)rows, nz);
    const int nruns = rp.parts * rp.run_k;
    if (nruns > w.l.rl.nruns) return PRISM_ERR_INVALID_ARG;
    ScoreArgs sa = score_args(c, w, qs[0], ks[0], len);
    sa.src = src; sa.kappa = E; sa.radius = radius;
    sa.hist = w.rhist; sa.runs = w.runs; sa.run_cnt = w.run_cnt;
    sa.parts = rp.parts; sa.run_k = rp.run_k;
    sa.Spos = nz == 1 ? Spos : nullptr; sa.spos_stride = spos_stride;
    if (cut) {
        sa.glen = cut->glen; sa.glmax = cut->glmax; sa.shard_lo = cut->lo;
    }
    sa.nz = nz;
    sa.zruns = rows * (size_t)nruns * kRunCap; sa.zcnt = rows * (size_t)nruns;
    sa.zhist = rows * kHistBins;
    for (int z = 0; z < nz; ++z) {
        sa.qz[z] = qs[z];
        sa.kz[z] = ks[z];
    }
    // One layer whose parts all fit the GPU at once (one block per SM), one
    // run each: the rescoring blocks of a row select together (no second
    // kernel); otherwise the selection kernel reads the runs.  The blocks of a
    // row wait for one another, so each of them must find room on an SM.
    // Beside an anchor scan (a block on every SM) the full-size rescoring
    // block leaves no room for an attention block, and a row whose block
    // waits behind attention blocks stalls (measured: ~50 against ~22 us a
    // layer); the two-stage block (group sum) leaves room for one.  So the
    // group sum uses it while an anchor scan may be in flight (`alone`
    // false), the full-size block otherwise; the group maximum selects in
    // place only when alone.
    const bool sum_fmt = sa.agg == kAggSum && !sa.q2;
    if ((alone || sum_fmt) && nz == 1 && rp.run_k == 1 && rp.parts <= 256 && rp.parts == w.l.rl.parts1 &&
        (long long)rp.parts * (long long)rows <= num_sms()) {
        sa.fused = 1;
        sa.two_stages = alone ? 0 : 1;
        sa.row_bar = w.rbar;
        sa.bar_base = w.bar_arrivals;
        w.bar_arrivals += 2u * (uint32_t)rp.parts;
        sa.part_cnt = w.part_cnt;
        sa.sel_out = outs[0];
        sa.kap_out = c.kappa;
        sa.tie_spill = w.ties;
        sa.tie_cap = w.l.rl.tie_cap;
        return cuda_status(launch_refine_rescore(sa, s));
    }
    // A grid of more blocks than SMs runs in waves of one full-size block per
    // SM; two two-stage blocks fit an SM, which halves the waves.
    if (sum_fmt && (long long)rp.parts * (long long)rows * nz > num_sms()) sa.two_stages = 1;
    PRISM_CUDA(launch_refine_rescore(sa, s));
    RunSelectArgs se{};
    se.runs = w.runs; se.run_cnt = w.run_cnt; se.nruns = nruns;
    se.hist = w.rhist; se.len = len;
    se.B = c.batch; se.Hkv = c.n_kv_heads; se.Lmax = c.max_len; se.kappa = c.kappa;
    se.tie_spill = w.ties; se.tie_cap = w.l.rl.tie_cap;
    se.nz = nz; se.zruns = sa.zruns; se.zcnt = sa.zcnt; se.zhist = sa.zhist;
    se.ztie = rows * (size_t)w.l.rl.tie_cap;
    for (int z = 0; z < nz; ++z) se.outz[z] = outs[z];
    se.idx_out = outs[0];
    se.st = w.st;
    return cuda_status(launch_select_runs(se, s));
}

// One refined layer: Eq. (5) over the +-r proposal (pool mode: the pool) of
// the canonical source selection `src`, then Eq. (6).
prism_status_t run_refine(const prism_config_t &c, const Ws &w, const void *q, const void *k,
                          const int32_t *len, const int32_t *src, int32_t *idx_out,
                          cudaStream_t s, float *Spos = nullptr, bool alone = true) {
    const void *qs[1] = {q};
    const void *ks[1] = {k};
    int32_t *outs[1] = {idx_out};
    return run_refine_batch(c, w, qs, ks, outs, 1, len, src, src_kappa_of(c), refine_radius_of(c),
                            Spos, c.max_len, s, alone);
}

prism_status_t run_attn(const prism_config_t &c, const Ws &w, const void *q, const void *k,
                        const void *v, const int32_t *len, const int32_t *idx, int idx_stride,
                        int n_idx, void *out, cudaStream_t s, float *cp_part = nullptr) {
    AttnArgs aa{};
    aa.q = q; aa.k = k; aa.v = v; aa.len = len; aa.idx = idx;
    aa.idx_stride = idx_stride; aa.n_idx = n_idx;
    aa.B = c.batch; aa.Hkv = c.n_kv_heads; aa.G = c.n_q_heads / c.n_kv_heads;
    aa.d = c.head_dim; aa.Lmax = c.max_len; aa.scale = eff_scale(c);
    aa.part_acc = w.pacc; aa.part_ml = w.pml; aa.ctl = w.attn_ctl; aa.out = out; aa.st = w.st;
    aa.cp_part = cp_part;
    return cuda_status(launch_sparse_attn(aa, s));
}

// The decode step's launch sequence.  With hp == nullptr everything goes to
// `s0`; otherwise the three streams of the DAG described at the top.  Every
// event is recorded (on the host) before any wait on it is enqueued.
prism_status_t enqueue_step(const prism_config_t &c, const Ws &w, const void *q,
                            const void *const *k, const void *const *v,
                            const void *const *kq, const int32_t *len,
                            void *out, int32_t *idx_out, cudaStream_t s0, DeviceHelpers *hp) {
    const int N = c.n_layers;
    const size_t rows = (size_t)c.batch * c.n_kv_heads;
    const size_t sel_elems = rows * (size_t)c.kappa;
    const size_t q_elems = (size_t)c.batch * c.n_q_heads * c.head_dim;
    const uint16_t *qb = static_cast<const uint16_t *>(q);
    uint16_t *ob = static_cast<uint16_t *>(out);
    int32_t *idx_base = idx_out ? idx_out : w.idx_all;
    // Pool mode: each anchor's pool, by layer.
    const bool pool = pool_mode(c);
    const size_t pool_elems = rows * (size_t)src_kappa_of(c);
    // Layer kinds: 1 anchor (F), 0 the mode's other layer (R), 2 shared (S,
    // Table 9: keeps the previous layer's selection).
    auto kind_of = [&](int l) { return c.mode == PRISM_MODE_DENSE_ANCHOR ? 1 : (int)c.anchor_mask[l]; };
    auto is_anchor = [&](int l) { return kind_of(l) == 1; };
    auto is_shared = [&](int l) { return kind_of(l) == 2; };
    std::vector<int> anchors;
    for (int l = 0; l < N; ++l)
        if (is_anchor(l)) anchors.push_back(l);
    const int NA = (int)anchors.size();

    cudaStream_t sA = hp ? hp->anchor : s0, sM = hp ? hp->chain : s0, sC = hp ? hp->attn : s0;
    cudaStream_t sX = hp ? hp->aux : s0;
    // Events: fork, two joins, per anchor "indexed" and "reached by the chain",
    // per layer "selected".
    cudaEvent_t ev_fork = nullptr, ev_join_m = nullptr, ev_join_c = nullptr;
    const cudaEvent_t *ev_indexed = nullptr, *ev_reached = nullptr, *ev_sel = nullptr;
    // pool mode: an anchor's scores done, its pool selected, its own top-kappa selected
    const cudaEvent_t *ev_scored = nullptr, *ev_pool = nullptr, *ev_kdone = nullptr;
    cudaEvent_t ev_join_x = nullptr;
    if (hp) {
        const cudaEvent_t *e = hp->events.data();
        ev_fork = e[0];
        ev_join_m = e[1];
        ev_join_c = e[2];
        ev_join_x = e[3];
        ev_indexed = e + 4;
        ev_reached = ev_indexed + NA;
        ev_sel = ev_reached + NA;
        ev_scored = ev_sel + N;
        ev_pool = ev_scored + NA;
        ev_kdone = ev_pool + NA;
    }

    PRISM_TRY(zero_control(w, s0));
    if (hp) {
        PRISM_CUDA(cudaEventRecord(ev_fork, s0));
        PRISM_CUDA(cudaStreamWaitEvent(sA, ev_fork, 0));
        PRISM_CUDA(cudaStreamWaitEvent(sM, ev_fork, 0));
        PRISM_CUDA(cudaStreamWaitEvent(sC, ev_fork, 0));
        PRISM_CUDA(cudaStreamWaitEvent(sX, ev_fork, 0));
    }
    // Pool mode with helper streams: the anchor stream only scans (Eq. (9));
    // the pool and the anchor's own top-kappa are selected on the aux stream,
    // so that they overlap the next anchor's scan.  Neither selection clears
    // the slot's histogram; the anchor stream clears it before the slot's
    // next scan, once both selections of the slot's previous anchor are done.
    auto index_anchor_pool = [&](int g) -> prism_status_t {
        const int l = anchors[g];
        const int slot = g % kAnchorAhead;
        if (g >= kAnchorAhead) {
            PRISM_CUDA(cudaStreamWaitEvent(sA, ev_reached[g - kAnchorAhead], 0));
            PRISM_CUDA(cudaStreamWaitEvent(sA, ev_kdone[g - kAnchorAhead], 0));
            PRISM_CUDA(cudaMemsetAsync(w.slot[slot].hist, 0, rows * kHistBins * sizeof(uint32_t), sA));
        }
        PRISM_TRY(run_anchor_score(c, w, slot, qb + (size_t)l * q_elems, kq ? kq[l] : k[l], len,
                                   nullptr, sA));
        PRISM_CUDA(cudaEventRecord(ev_scored[g], sA));
        PRISM_CUDA(cudaStreamWaitEvent(sX, ev_scored[g], 0));
        const Slot &sl = w.slot[slot];
        SelectArgs p = select_args(c, w, sl, len, w.pool_all + (size_t)l * pool_elems);
        p.kappa = src_kappa_of(c);
        p.radius = 0;
        p.keep_hist = 1;
        PRISM_CUDA(launch_select(p, sX));
        PRISM_CUDA(cudaEventRecord(ev_pool[g], sX));
        SelectArgs t = select_args(c, w, sl, len, idx_base + (size_t)l * sel_elems);
        t.keep_hist = 1;
        PRISM_CUDA(launch_select(t, sX));
        PRISM_CUDA(cudaEventRecord(ev_kdone[g], sX));
        return PRISM_OK;
    };
    // An anchor's scoring and selection depend on nothing but its own q and K,
    // so both run on the anchor stream, kAnchorAhead anchors ahead of the
    // chain of refined layers (the anchor slots form a ring of that size).
    auto index_anchor = [&](int g) -> prism_status_t {
        if (pool && hp) return index_anchor_pool(g);
        const int l = anchors[g];
        if (hp && g >= kAnchorAhead) PRISM_CUDA(cudaStreamWaitEvent(sA, ev_reached[g - kAnchorAhead], 0));
        PRISM_TRY(run_anchor_score(c, w, g % kAnchorAhead, qb + (size_t)l * q_elems,
                                   kq ? kq[l] : k[l], len,
                                   nullptr, sA));
        if (pool) {
            PRISM_TRY(run_pool_select(c, w, g % kAnchorAhead, len, w.pool_all + (size_t)l * pool_elems,
                                      idx_base + (size_t)l * sel_elems, sA));
        } else {
            PRISM_TRY(run_anchor_select(c, w, g % kAnchorAhead, len, idx_base + (size_t)l * sel_elems,
                                        sA));
        }
        if (hp) PRISM_CUDA(cudaEventRecord(ev_indexed[g], sA));
        return PRISM_OK;
    };
    if (hp) {
        for (int g = 0; g < NA && g < kAnchorAhead; ++g) PRISM_TRY(index_anchor(g));
    }

    const int32_t *anchor_sel = nullptr, *prev_sel = nullptr;
    int anchor_layer = 0;
    std::vector<char> batched(pool ? (size_t)N : 0, 0);   // pool mode: refined layers enqueued
    bool prev_is_anchor_sel = false;     // the previous layer's selection is an anchor's own
    int g = 0;
    for (int l = 0; l < N; ++l) {
        const void *ql = qb + (size_t)l * q_elems;
        const int32_t *src = c.chain == PRISM_CHAIN_ANCHOR ? anchor_sel : prev_sel;
        int32_t *dst = idx_base + (size_t)l * sel_elems;
        const int32_t *cur = dst;
        if (is_anchor(l)) {
            if (hp) {
                PRISM_CUDA(cudaStreamWaitEvent(sM, pool ? ev_pool[g] : ev_indexed[g], 0));
                PRISM_CUDA(cudaEventRecord(ev_reached[g], sM));
                if (g + kAnchorAhead < NA) PRISM_TRY(index_anchor(g + kAnchorAhead));
            } else {
                PRISM_TRY(index_anchor(g));
            }
            anchor_sel = dst;
            anchor_layer = l;
            ++g;
        } else if (is_shared(l)) {
            // Table 9's shared layer: the previous layer's selection, unchanged.
            // In pool mode an anchor's own selection comes from the aux
            // stream, so a copy of it waits for that selection.
            if (pool && hp && prev_is_anchor_sel) PRISM_CUDA(cudaStreamWaitEvent(sM, ev_kdone[g - 1], 0));
            if (idx_out) {
                PRISM_CUDA(cudaMemcpyAsync(dst, prev_sel, sel_elems * sizeof(int32_t),
                                           cudaMemcpyDeviceToDevice, sM));
            } else {
                cur = prev_sel;
            }
        } else if (pool) {
            // Eq. (5)-(6) over the nearest preceding anchor's pool.  The
            // refined layers of a group depend on that pool alone, so up to
            // kMaxZ of them (skipping shared layers) are rescored and selected
            // by one launch each, enqueued at the first of them.
            if (!batched[l]) {
                const void *qs[kMaxZ];
                const void *ks[kMaxZ];
                int32_t *outs[kMaxZ];
                int nz = 0;
                for (int e = l; e < N && !is_anchor(e) && nz < kMaxZ; ++e) {
                    if (is_shared(e)) continue;
                    qs[nz] = qb + (size_t)e * q_elems;
                    ks[nz] = kq ? kq[e] : k[e];
                    outs[nz] = idx_base + (size_t)e * sel_elems;
                    batched[e] = 1;
                    ++nz;
                }
                PRISM_TRY(run_refine_batch(c, w, qs, ks, outs, nz, len,
                                           w.pool_all + (size_t)anchor_layer * pool_elems,
                                           src_kappa_of(c), 0, nullptr, 0, sM, !hp || g >= NA));
            }
        } else if (c.mode == PRISM_MODE_STATIC_REUSE) {
            if (idx_out) {
                PRISM_CUDA(cudaMemcpyAsync(dst, src, sel_elems * sizeof(int32_t),
                                           cudaMemcpyDeviceToDevice, sM));
            } else {
                cur = src;
            }
        } else {
            // alone: on one stream, or once no anchor scan remains ahead of the
            // chain (it picks the rescoring block size; see run_refine_batch).
            // (A schedule that ran every group's refined layers alone,
            // the next anchor's scan overlapping only the current anchor's
            // selection, was measured slower: 38.7 against 30.6 us a layer at
            // 128K; the scans' streaming then no longer hides under the
            // refined layers' latency-bound phases.)
            PRISM_TRY(run_refine(c, w, ql, k[l], len, src, dst, sM, nullptr, !hp || g >= NA));
        }
        if (hp) {
            PRISM_CUDA(cudaEventRecord(ev_sel[l], sM));
            PRISM_CUDA(cudaStreamWaitEvent(sC, ev_sel[l], 0));
            // a pool-mode anchor's own selection comes from the aux stream
            if (pool && is_anchor(l)) PRISM_CUDA(cudaStreamWaitEvent(sC, ev_kdone[g - 1], 0));
        }
        PRISM_TRY(run_attn(c, w, ql, k[l], v[l], len, cur, c.kappa, c.kappa,
                           ob + (size_t)l * q_elems, sC));
        prev_sel = cur;
        if (!is_shared(l)) prev_is_anchor_sel = is_anchor(l);
    }
    if (hp) {
        // Every anchor score was waited on by M; join M and C into the caller's stream.
        PRISM_CUDA(cudaEventRecord(ev_join_m, sM));
        PRISM_CUDA(cudaEventRecord(ev_join_c, sC));
        PRISM_CUDA(cudaEventRecord(ev_join_x, sX));
        PRISM_CUDA(cudaStreamWaitEvent(s0, ev_join_m, 0));
        PRISM_CUDA(cudaStreamWaitEvent(s0, ev_join_c, 0));
        PRISM_CUDA(cudaStreamWaitEvent(s0, ev_join_x, 0));
    }
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
    PRISM_TRY(run_anchor_score(*cfg, w, 0, q, k, len, nullptr, s));
    PRISM_TRY(run_anchor_select(*cfg, w, 0, len, idx_out, s));
    if (scores_out) {
        // The selection reads the workspace copy (its staged copies may round
        // a row's end up to 16 bytes); the caller gets the scores afterwards.
        const size_t bytes = (size_t)cfg->batch * cfg->n_kv_heads * cfg->max_len * sizeof(float);
        PRISM_CUDA(cudaMemcpyAsync(scores_out, w.slot[0].S, bytes, cudaMemcpyDeviceToDevice, s));
    }
    return PRISM_OK;
}

prism_status_t prism_index_pool(const prism_config_t *cfg, const void *q, const void *k,
                                const int32_t *len, int32_t *pool_out, int32_t *idx_out,
                                float *scores_out, void *ws, size_t ws_bytes, void *stream) {
    PRISM_TRY(check_config(cfg));
    if (cfg->mode != PRISM_MODE_POOL) return PRISM_ERR_INVALID_ARG;
    if (!q || !k || !len || !pool_out || !idx_out || pool_out == idx_out) return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(len, 4) || !aligned(pool_out, 4) ||
        !aligned(idx_out, 4) || (scores_out && !aligned(scores_out, 4)))
        return PRISM_ERR_INVALID_ARG;
    Ws w;
    PRISM_TRY(carve(*cfg, ws, ws_bytes, &w));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PRISM_TRY(zero_control(w, s));
    PRISM_TRY(run_anchor_score(*cfg, w, 0, q, k, len, nullptr, s));
    PRISM_TRY(run_pool_select(*cfg, w, 0, len, pool_out, idx_out, s));
    if (scores_out) {
        const size_t bytes = (size_t)cfg->batch * cfg->n_kv_heads * cfg->max_len * sizeof(float);
        PRISM_CUDA(cudaMemcpyAsync(scores_out, w.slot[0].S, bytes, cudaMemcpyDeviceToDevice, s));
    }
    return PRISM_OK;
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
    return run_anchor_score(*cfg, w, 0, q, k, len, scores_out, static_cast<cudaStream_t>(stream));
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
    CanonArgs ca{};
    ca.idx = idx_prev; ca.len = len; ca.B = cfg->batch; ca.Hkv = cfg->n_kv_heads;
    ca.Lmax = cfg->max_len; ca.kappa = src_kappa_of(*cfg);
    ca.radius = refine_radius_of(*cfg);
    ca.out = w.canon; ca.out_off = nullptr; ca.st = w.st;
    PRISM_CUDA(launch_canonicalize(ca, s));
    // With an export, the rescoring also leaves every candidate's score by
    // position in anchor slot 0 (unused by this call).
    float *Spos = all ? w.slot[0].S : nullptr;
    PRISM_TRY(run_refine(*cfg, w, q, k, len, w.canon, idx_out, s, Spos));
    if (all)
        PRISM_CUDA(launch_export_candidates(w.canon, src_kappa_of(*cfg), refine_radius_of(*cfg), len,
                                            cfg->batch, cfg->n_kv_heads, cfg->max_len, Spos,
                                            cand_pos, cand_score, cand_count, cand_cap, w.st, s));
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    PRISM_CUDA(cudaMemsetAsync(w.attn_ctl, 0,
                               (size_t)cfg->batch * cfg->n_kv_heads * sizeof(RowCtl), s));
    return run_attn(*cfg, w, q, k, v, len, idx, n_idx, n_idx, out, s);
}

prism_status_t prism_sparse_decode_noalloc(const prism_config_t *cfg, const void *q,
                                           const void *k, const void *v, const int32_t *len,
                                           const int32_t *idx, int32_t n_idx, void *out,
                                           void *stream) {
    PRISM_TRY(check_config(cfg));
    if (!q || !k || !v || !len || !idx || !out) return PRISM_ERR_INVALID_ARG;
    if (n_idx < 1 || n_idx > cfg->kappa) return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(len, 4) || !aligned(idx, 4))
        return PRISM_ERR_INVALID_ARG;
    const long long rows = (long long)cfg->batch * cfg->n_kv_heads;
    const long long nsplit = (n_idx + kAttnChunk - 1) / kAttnChunk;
    const long long G = cfg->n_q_heads / cfg->n_kv_heads;
    if (rows > kStaticAttnMaxRows ||
        rows * nsplit * G * cfg->head_dim > (long long)kStaticAttnMaxAccFloats)
        return PRISM_ERR_WORKSPACE;
    StaticAttnScratch sc;
    PRISM_CUDA(static_attn_scratch(&sc));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The merge counters must start at zero (the kernel leaves them zeroed,
    // but a call cut short would not).
    PRISM_CUDA(cudaMemsetAsync(sc.st, 0, sizeof(DevStatus), s));
    PRISM_CUDA(cudaMemsetAsync(sc.ctl, 0, (size_t)rows * sizeof(RowCtl), s));
    AttnArgs aa{};
    aa.q = q; aa.k = k; aa.v = v; aa.len = len; aa.idx = idx;
    aa.idx_stride = n_idx; aa.n_idx = n_idx;
    aa.B = cfg->batch; aa.Hkv = cfg->n_kv_heads; aa.G = (int)G;
    aa.d = cfg->head_dim; aa.Lmax = cfg->max_len; aa.scale = eff_scale(*cfg);
    aa.part_acc = sc.part_acc; aa.part_ml = sc.part_ml; aa.ctl = sc.ctl; aa.out = out; aa.st = sc.st;
    return cuda_status(launch_sparse_attn(aa, s));
}

static prism_status_t decode_step_impl(const prism_config_t *cfg, const void *q,
                                       const void *const *k, const void *const *v,
                                       const void *const *kq, const int32_t *len, void *out,
                                       int32_t *idx_out, void *ws, size_t ws_bytes, void *stream) {
    PRISM_TRY(check_config(cfg));
    const prism_config_t &c = *cfg;
    if (c.n_layers < 1 || !q || !k || !v || !len || !out) return PRISM_ERR_INVALID_ARG;
    // the 2-bit keys come with their own call (the step needs both caches)
    if (((c.flags & PRISM_FLAG_INT2_KEYS) != 0) != (kq != nullptr)) return PRISM_ERR_INVALID_ARG;
    if (c.mode != PRISM_MODE_DENSE_ANCHOR) {
        // layer kinds: 0 refined, 1 anchor, 2 shared; layer 0 is an anchor
        if (!c.anchor_mask || c.anchor_mask[0] != 1) return PRISM_ERR_INVALID_ARG;
        for (int l = 0; l < c.n_layers; ++l)
            if (c.anchor_mask[l] > 2) return PRISM_ERR_INVALID_ARG;
    }
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(len, 4) ||
        (idx_out && !aligned(idx_out, 4)))
        return PRISM_ERR_INVALID_ARG;
    for (int l = 0; l < c.n_layers; ++l) {
        if (!k[l] || !v[l] || !aligned(k[l], 16) || !aligned(v[l], 16)) return PRISM_ERR_INVALID_ARG;
        if (kq && (!kq[l] || !aligned(kq[l], 16))) return PRISM_ERR_INVALID_ARG;
    }
    Ws w;
    PRISM_TRY(carve(c, ws, ws_bytes, &w));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c.flags & PRISM_FLAG_SERIAL)
        return enqueue_step(c, w, q, k, v, kq, len, out, idx_out, s, nullptr);
    std::lock_guard<std::mutex> lock(g_helpers_mu);
    DeviceHelpers *hp = nullptr;
    PRISM_TRY(helpers_for_current_device(4 + 6 * (size_t)c.n_layers, &hp));
    return enqueue_step(c, w, q, k, v, kq, len, out, idx_out, s, hp);
}

prism_status_t prism_decode_step(const prism_config_t *cfg, const void *q, const void *const *k,
                                 const void *const *v, const int32_t *len, void *out,
                                 int32_t *idx_out, void *ws, size_t ws_bytes, void *stream) {
    return decode_step_impl(cfg, q, k, v, nullptr, len, out, idx_out, ws, ws_bytes, stream);
}

prism_status_t prism_decode_step_kq(const prism_config_t *cfg, const void *q,
                                    const void *const *k, const void *const *v,
                                    const void *const *kq, const int32_t *len, void *out,
                                    int32_t *idx_out, void *ws, size_t ws_bytes, void *stream) {
    if (!kq) return PRISM_ERR_INVALID_ARG;
    return decode_step_impl(cfg, q, k, v, kq, len, out, idx_out, ws, ws_bytes, stream);
}

prism_status_t prism_quantize_keys(const prism_config_t *cfg, const void *k, const int32_t *len,
                                   int32_t start, void *kq, void *ws, size_t ws_bytes,
                                   void *stream) {
    PRISM_TRY(check_config(cfg));
    if (!k || !len || !kq || start < 0) return PRISM_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(kq, 16) || !aligned(len, 4)) return PRISM_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, 256) || ws_bytes < sizeof(DevStatus)) return PRISM_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_keys(k, len, cfg->batch, cfg->n_kv_heads, cfg->head_dim,
                                            cfg->max_len, start, kq, static_cast<DevStatus *>(ws),
                                            static_cast<cudaStream_t>(stream)));
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

int32_t prism_version(void) { return 10200; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Context-parallel pieces (include/prism_cp.h).  A rank's workspace starts
// with the single-GPU layout of its shard (capacity shard_len, one layer),
// followed by the buffers of the shard-local steps and of the merge.
namespace {

prism_config_t local_config(const prism_config_t &c, const prism_cp_shard_t &sh) {
    prism_config_t lc = c;
    lc.max_len = sh.shard_len;
    lc.n_layers = 1;
    lc.anchor_mask = nullptr;
    return lc;
}

struct CpLayout {
    Layout l;
    int kmax, R, cs_m;
    size_t llen, lsel, lpool, latt;
    size_t mS, mcpos, mcount, mhist, mspill, total;
};

CpLayout make_cp_layout(const prism_config_t &c, const prism_cp_shard_t &sh) {
    CpLayout L{};
    const size_t rows = (size_t)c.batch * c.n_kv_heads;
    // a refined layer rescores its proposal cut to the shard, from the global source
    L.l = make_layout(local_config(c, sh));
    L.kmax = src_kappa_of(c);
    L.R = sh.n_ranks;
    L.cs_m = (int)(((long long)L.R * L.kmax + 3) & ~3LL);
    size_t off = L.l.total;
    L.llen = off;     off = align256(off + (size_t)c.batch * sizeof(int32_t));
    L.lsel = off;     off = align256(off + rows * (size_t)c.kappa * sizeof(int32_t));
    L.lpool = off;    off = align256(off + rows * (size_t)L.kmax * sizeof(int32_t));
    L.latt = off;     off = align256(off + rows * (size_t)c.kappa * sizeof(int32_t));
    L.mS = off;       off = align256(off + rows * (size_t)L.cs_m * sizeof(float));
    L.mcpos = off;    off = align256(off + rows * (size_t)L.cs_m * sizeof(int32_t));
    L.mcount = off;   off = align256(off + rows * ((size_t)L.R * L.kmax + 1) * sizeof(int32_t));
    L.mhist = off;    off = align256(off + rows * kHistBins * sizeof(uint32_t));
    L.mspill = off;   off = align256(off + rows * 2 * (size_t)L.cs_m * sizeof(uint64_t));
    L.total = off;
    return L;
}

prism_status_t check_cp(const prism_config_t *c, const prism_cp_shard_t *sh) {
    PRISM_TRY(check_config(c));
    if (!sh) return PRISM_ERR_INVALID_ARG;
    if (sh->n_ranks < 1 || sh->rank < 0 || sh->rank >= sh->n_ranks || sh->shard_len < 1)
        return PRISM_ERR_INVALID_ARG;
    // the shards cover the capacity; a shard's positions (up to
    // n_ranks * shard_len) must fit the 32-bit positions of the kernels
    if ((long long)sh->n_ranks * sh->shard_len < c->max_len) return PRISM_ERR_INVALID_ARG;
    if ((long long)sh->n_ranks * sh->shard_len > INT32_MAX) return PRISM_ERR_INVALID_ARG;
    if (c->flags & PRISM_FLAG_INT2_KEYS) return PRISM_ERR_UNSUPPORTED;
    if (sh->shard_len > PRISM_MAX_LEN) return PRISM_ERR_UNSUPPORTED;
    if ((long long)sh->n_ranks * src_kappa_of(*c) > PRISM_MAX_LEN) return PRISM_ERR_UNSUPPORTED;
    return PRISM_OK;
}

struct CpWs {
    Ws w;
    CpLayout L;
    int32_t *llen, *lsel, *lpool, *latt;
    float *mS;
    int32_t *mcpos, *mcount;
    uint32_t *mhist;
    uint64_t *mspill;
};

prism_status_t carve_cp(const prism_config_t &c, const prism_cp_shard_t &sh, void *ws,
                        size_t ws_bytes, CpWs *x) {
    if (!ws || !aligned(ws, 256)) return PRISM_ERR_INVALID_ARG;
    x->L = make_cp_layout(c, sh);
    if (ws_bytes < x->L.total) return PRISM_ERR_WORKSPACE;
    PRISM_TRY(carve(local_config(c, sh), ws, ws_bytes, &x->w));
    uint8_t *b = static_cast<uint8_t *>(ws);
    x->llen = reinterpret_cast<int32_t *>(b + x->L.llen);
    x->lsel = reinterpret_cast<int32_t *>(b + x->L.lsel);
    x->lpool = reinterpret_cast<int32_t *>(b + x->L.lpool);
    x->latt = reinterpret_cast<int32_t *>(b + x->L.latt);
    x->mS = reinterpret_cast<float *>(b + x->L.mS);
    x->mcpos = reinterpret_cast<int32_t *>(b + x->L.mcpos);
    x->mcount = reinterpret_cast<int32_t *>(b + x->L.mcount);
    x->mhist = reinterpret_cast<uint32_t *>(b + x->L.mhist);
    x->mspill = reinterpret_cast<uint64_t *>(b + x->L.mspill);
    return PRISM_OK;
}

CpPrepArgs cp_prep_args(const prism_config_t &c, const prism_cp_shard_t &sh, const CpWs &x,
                        const int32_t *len) {
    CpPrepArgs pa{};
    pa.what = kCpPrepLen;
    pa.len = len;
    pa.B = c.batch; pa.Hkv = c.n_kv_heads; pa.Lmax = c.max_len;
    pa.lo = sh.rank * sh.shard_len; pa.cap = sh.shard_len;
    pa.llen = x.llen; pa.st = x.w.st;
    return pa;
}

prism_status_t cp_pack(const prism_config_t &c, const prism_cp_shard_t &sh, const int32_t *sel,
                       int n, const float *S, int32_t *pos_out, float *score_out,
                       cudaStream_t s) {
    CpPackArgs pk{};
    pk.sel = sel; pk.rows = c.batch * c.n_kv_heads; pk.n = n; pk.lo = sh.rank * sh.shard_len;
    pk.S = S; pk.sstride = sh.shard_len;
    pk.pos_out = pos_out; pk.score_out = score_out;
    return cuda_status(launch_cp_pack(pk, s));
}

}  // namespace

extern "C" {

prism_status_t prism_cp_workspace_size(const prism_config_t *cfg, const prism_cp_shard_t *shard,
                                       size_t *bytes) {
    PRISM_TRY(check_cp(cfg, shard));
    if (!bytes) return PRISM_ERR_INVALID_ARG;
    *bytes = make_cp_layout(*cfg, *shard).total;
    return PRISM_OK;
}

prism_status_t prism_cp_index_local(const prism_config_t *cfg, const prism_cp_shard_t *shard,
                                    const void *q, const void *k, const int32_t *len,
                                    const int32_t *src, int32_t *cand_pos, float *cand_score,
                                    int32_t *pool_pos, float *pool_score, void *ws,
                                    size_t ws_bytes, void *stream) {
    PRISM_TRY(check_cp(cfg, shard));
    if (!q || !k || !len || !cand_pos || !cand_score) return PRISM_ERR_INVALID_ARG;
    const bool pool = pool_mode(*cfg);
    const bool want_pool = pool && !src;
    if (want_pool != (pool_pos != nullptr) || want_pool != (pool_score != nullptr))
        return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(len, 4) || !aligned(cand_pos, 4) ||
        !aligned(cand_score, 4) || (src && !aligned(src, 4)) ||
        (pool_pos && !aligned(pool_pos, 4)) || (pool_score && !aligned(pool_score, 4)))
        return PRISM_ERR_INVALID_ARG;
    CpWs x;
    PRISM_TRY(carve_cp(*cfg, *shard, ws, ws_bytes, &x));
    const prism_config_t lc = local_config(*cfg, *shard);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CpPrepArgs pa = cp_prep_args(*cfg, *shard, x, len);
    PRISM_CUDA(launch_cp_prepare(pa, s));
    // A plain stream operation between the kernel above and the ones below:
    // those may read the shard lengths before their grid-dependency wait.
    PRISM_TRY(zero_control(x.w, s));
    if (!src) {
        PRISM_TRY(run_anchor_score(lc, x.w, 0, q, k, x.llen, nullptr, s));
        if (pool)
            PRISM_TRY(run_pool_select(lc, x.w, 0, x.llen, x.lpool, x.lsel, s));
        else
            PRISM_TRY(run_anchor_select(lc, x.w, 0, x.llen, x.lsel, s));
        PRISM_TRY(cp_pack(*cfg, *shard, x.lsel, cfg->kappa, x.w.slot[0].S, cand_pos,
                          cand_score, s));
        if (pool)
            PRISM_TRY(cp_pack(*cfg, *shard, x.lpool, src_kappa_of(*cfg), x.w.slot[0].S, pool_pos,
                              pool_score, s));
        return PRISM_OK;
    }
    // Eq. (5)-(6) over the proposal of the global source cut to the shard;
    // the candidates' scores are left by local position in slot 0 for the pack.
    const void *qs[1] = {q};
    const void *ks[1] = {k};
    int32_t *outs[1] = {x.lsel};
    const CutToShard cut{len, cfg->max_len, shard->rank * shard->shard_len};
    PRISM_TRY(run_refine_batch(lc, x.w, qs, ks, outs, 1, x.llen, src, src_kappa_of(*cfg),
                               refine_radius_of(*cfg), x.w.slot[0].S, shard->shard_len, s, true,
                               &cut));
    return cp_pack(*cfg, *shard, x.lsel, cfg->kappa, x.w.slot[0].S, cand_pos, cand_score, s);
}

prism_status_t prism_cp_merge(const prism_config_t *cfg, const prism_cp_shard_t *shard,
                              int32_t n_out, const int32_t *cand_pos, const float *cand_score,
                              const int32_t *len, int32_t *idx_out, void *ws, size_t ws_bytes,
                              void *stream) {
    PRISM_TRY(check_cp(cfg, shard));
    if (!cand_pos || !cand_score || !len || !idx_out) return PRISM_ERR_INVALID_ARG;
    if (n_out != cfg->kappa && !(pool_mode(*cfg) && n_out == src_kappa_of(*cfg)))
        return PRISM_ERR_INVALID_ARG;
    if (!aligned(cand_pos, 4) || !aligned(cand_score, 4) || !aligned(len, 4) ||
        !aligned(idx_out, 4))
        return PRISM_ERR_INVALID_ARG;
    CpWs x;
    PRISM_TRY(carve_cp(*cfg, *shard, ws, ws_bytes, &x));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int R = shard->n_ranks;
    if (R == 1) {
        // One shard: its list (ascending, -1 padded, n_out entries a row) is
        // the selection.
        return cuda_status(cudaMemcpyAsync(idx_out, cand_pos,
                                           (size_t)cfg->batch * cfg->n_kv_heads * n_out * sizeof(int32_t),
                                           cudaMemcpyDeviceToDevice, s));
    }
    CpMergeArgs ma{};
    ma.pos = cand_pos; ma.score = cand_score;
    ma.R = R; ma.rows = cfg->batch * cfg->n_kv_heads; ma.n = n_out;
    ma.B = cfg->batch; ma.Hkv = cfg->n_kv_heads; ma.Lmax = cfg->max_len; ma.len = len;
    ma.S = x.mS; ma.cpos = x.mcpos; ma.cstride = x.L.cs_m; ma.count_out = x.mcount;
    ma.hist = x.mhist; ma.st = x.w.st;
    PRISM_CUDA(launch_cp_merge_prepare(ma, s));
    SelectArgs se = select_args(*cfg, x.w, x.w.slot[0], len, idx_out);
    se.S = x.mS; se.cpos = x.mcpos; se.src_off = x.mcount;
    se.kappa = n_out; se.radius = 0;
    se.src_kappa = R * n_out; se.n_bound = R * n_out;
    se.cstride = x.L.cs_m; se.hist = x.mhist; se.cspill = x.mspill;
    return cuda_status(launch_select(se, s));
}

prism_status_t prism_cp_attn_local(const prism_config_t *cfg, const prism_cp_shard_t *shard,
                                   const void *q, const void *k, const void *v,
                                   const int32_t *len, const int32_t *idx, float *part_out,
                                   void *ws, size_t ws_bytes, void *stream) {
    PRISM_TRY(check_cp(cfg, shard));
    if (!q || !k || !v || !len || !idx || !part_out) return PRISM_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(len, 4) ||
        !aligned(idx, 4) || !aligned(part_out, 4))
        return PRISM_ERR_INVALID_ARG;
    CpWs x;
    PRISM_TRY(carve_cp(*cfg, *shard, ws, ws_bytes, &x));
    const prism_config_t lc = local_config(*cfg, *shard);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CpPrepArgs pa = cp_prep_args(*cfg, *shard, x, len);
    pa.what = kCpPrepSelection;
    pa.src = idx; pa.src_kappa = cfg->kappa;
    pa.out = x.latt; pa.out_kappa = cfg->kappa;
    PRISM_CUDA(launch_cp_prepare(pa, s));
    // plain stream operation (see prism_cp_index_local), and the attention's row counters
    PRISM_CUDA(cudaMemsetAsync(x.w.attn_ctl, 0,
                               (size_t)cfg->batch * cfg->n_kv_heads * sizeof(RowCtl), s));
    // the attention's row merge leaves this rank's partial (acc, m, l)
    return run_attn(lc, x.w, q, k, v, x.llen, x.latt, cfg->kappa, cfg->kappa, nullptr, s, part_out);
}

prism_status_t prism_cp_combine(const prism_config_t *cfg, int32_t n_ranks,
                                const float *part_all, void *out, void *stream) {
    PRISM_TRY(check_config(cfg));
    if (n_ranks < 1 || !part_all || !out) return PRISM_ERR_INVALID_ARG;
    if (!aligned(part_all, 4) || !aligned(out, 16)) return PRISM_ERR_INVALID_ARG;
    CpCombineArgs ca{};
    ca.part = part_all; ca.R = n_ranks;
    ca.heads = cfg->batch * cfg->n_q_heads; ca.d = cfg->head_dim; ca.out = out;
    return cuda_status(launch_cp_combine(ca, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
