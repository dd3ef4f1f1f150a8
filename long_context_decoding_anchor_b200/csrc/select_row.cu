// select_row.cu -- exact top-kappa selection (Eq. (2) and Eq. (6) of "Prism
// Attention", section 4.1) by ONE thread block per (batch, KV head) row, for
// rows of at most kRowMaxItems items and budgets of at most kRowMaxKappa.
//
// Items are a refined layer's candidates -- scores at proposal slots, the
// slots enumerating the proposal in ascending position order, with the
// position of each slot beside it -- or an anchor layer's scores by position.
// Either way a lower item index is a lower position, so the tie rule (lower
// position wins) is a rule on item indices.  Scores are compared through
// order-preserving 32-bit keys, so every decision is exact.
//
// The selected items are marked in a shared-memory bitmap over the row's item
// indices rather than gathered in order, so no step has to keep items sorted:
//   1. the row's 2048-bin histogram (built by the scoring kernel) gives the
//      first radix digit b1 of the kappa-th key; meanwhile the first scores
//      are already in flight (plain 16-byte loads into registers, one round
//      ahead of their use);
//   2. one pass marks every item of digit > b1 and lists the items of digit
//      b1 (the ties of the first digit, a few percent of the row);
//   3. the ties' next 11 bits are histogrammed: the second-level bin holding
//      the kappa-th key usually has a handful of items, which one warp ranks
//      directly (key descending, index ascending); a crowded bin falls back to
//      a 10-bit histogram and a radix select on the index.  The selected ties
//      are marked;
//   4. the bitmap is enumerated in word order (a block scan of popcounts): the
//      selection comes out in ascending position order, the positions of a
//      refined row read from its slot positions.  When asked, the enumeration
//      offsets of the +-r proposal around the new selection follow.
// No cluster, no distributed shared memory, no inter-block traffic: the row's
// scores (L2-resident, written just before) are read once.
#include "select_impl.cuh"

namespace prism {

constexpr int kRowThreads = 512;
constexpr int kRowU = 4;                             // 16-byte loads a thread per round
constexpr int kRowRound4 = kRowThreads * kRowU;       // float4 groups a round
constexpr int kRowTieCap = 4096;                     // first-digit ties kept in shared memory

struct RowShared {
    uint32_t hist[kHistBins];
    int scratch[2 * kSelMaxWarps + 8];
    int thr[2];
    int ntie;
    int n_small;
    uint64_t small[kSmallCap];
};

// Among the m items of first digit b1 (tie_at(e): key << 32 | index, the
// index breaking ties, lower first), marks the need1 best: those whose key
// (and index) rank within the first need1.  The second 11 bits usually leave
// a handful of items in the bin of the need1-th, which one warp ranks
// directly; a crowded bin falls back to a 10-bit histogram and a radix select
// on the index.  Whole block; contains __syncthreads() unless every tie is
// selected.
template <class SM, class TieAt, class Mark>
__device__ void mark_selected_ties(SM &sm, TieAt tie_at, Mark mark, int m, uint32_t b1, int need1) {
    const int tid = threadIdx.x, lane = tid & 31, nt = blockDim.x;
    if (m <= 0) return;
    if (need1 >= m) {
        for (int e = tid; e < m; e += nt) mark(tie_at(e));
        return;
    }
    zero_hist(sm, kHistBins);
    for (int e = tid; e < m; e += nt)
        atomicAdd(&sm.hist[((uint32_t)(tie_at(e) >> 32) >> 10) & 0x7ffu], 1u);
    if (tid == 0) sm.n_small = 0;
    __syncthreads();
    int b2, above2;
    threshold_bin(sm, kHistBins, need1, &b2, &above2);
    const int need2 = need1 - above2;
    const uint32_t hi21 = (b1 << 21) | ((uint32_t)b2 << 10);
    if ((int)sm.hist[b2] <= kSmallCap) {
        for (int e = tid; e < m; e += nt) {
            const uint64_t it = tie_at(e);
            const uint32_t k21 = (uint32_t)(it >> 32) & 0xfffffc00u;
            if (k21 > hi21) mark(it);
            else if (k21 == hi21) sm.small[atomicAdd(&sm.n_small, 1)] = it;
        }
        __syncthreads();
        if (tid < 32) {
            // rank = items ahead in (key descending, index ascending)
            const int ns = sm.n_small;
            for (int i = lane; i < ns; i += 32) {
                const uint64_t u = sm.small[i];
                const uint32_t ku = (uint32_t)(u >> 32);
                const uint32_t iu = (uint32_t)u;
                int rk = 0;
                for (int j = 0; j < ns; ++j) {
                    const uint64_t w = sm.small[j];
                    const uint32_t kw = (uint32_t)(w >> 32);
                    rk += kw > ku || (kw == ku && (uint32_t)w < iu);
                }
                if (rk < need2) mark(u);
            }
        }
    } else {
        uint32_t T;
        int cutoff;
        resolve_threshold(sm, tie_at, m, b1, need1, &T, &cutoff);
        for (int e = tid; e < m; e += nt) {
            const uint64_t it = tie_at(e);
            const uint32_t k_ = (uint32_t)(it >> 32);
            if (k_ > T || (k_ == T && (int)(uint32_t)it <= cutoff)) mark(it);
        }
    }
}

// Words of the selection bitmap for rows of up to `cap` items (a 16-byte skew
// of up to 3 items in front, whole rounds of loads).
__host__ __device__ inline int row_bitmap_words(int cap) {
    const int g4 = (cap + 3 + 3) / 4;
    const int rounds = (g4 + kRowRound4 - 1) / kRowRound4;
    return rounds * kRowRound4 / 8;
}
__host__ __device__ inline size_t row_select_smem(int cap, int kappa) {
    return (size_t)row_bitmap_words(cap) * 4 + (size_t)kRowTieCap * 8 + (size_t)kappa * 4;
}

__global__ void __maxnreg__(80) k_select_row(SelectArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ RowShared sm;
    const int cap = a.row_cap;
    uint32_t *bm = reinterpret_cast<uint32_t *>(dyn);
    uint64_t *ties = reinterpret_cast<uint64_t *>(dyn + (size_t)row_bitmap_words(cap) * 4);
    int32_t *sel = reinterpret_cast<int32_t *>(ties + kRowTieCap);
    const int row = blockIdx.y;
    const size_t z = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31;
    const int cstride = a.cstride > 0 ? a.cstride : a.Lmax;
    const bool refine = a.cpos != nullptr;
    const int src_kappa = a.src_kappa > 0 ? a.src_kappa : a.kappa;
    const float *Srow = a.S + z * a.zS + (size_t)row * cstride;
    const int32_t *cpos = refine ? a.cpos + z * a.zS + (size_t)row * cstride : nullptr;
    int32_t *out = (a.nz > 1 ? a.outz[z] : a.idx_out) + (size_t)row * a.kappa;
    uint64_t *tie_g = a.cspill + z * a.zspill + (size_t)row * 2 * cstride + cstride;
    uint32_t *hist_g = a.hist + z * a.zhist + (size_t)row * kHistBins;
    // Item i sits in float4 group (i + skew) / 4 of the 16-byte aligned view.
    const int skew = (int)((reinterpret_cast<uintptr_t>(Srow) & 15) >> 2);
    const float4 *S4 = reinterpret_cast<const float4 *>(reinterpret_cast<uintptr_t>(Srow) & ~(uintptr_t)15);
    const int cap4 = (skew + min(cap, cstride) + 3) >> 2;    // groups inside the row's buffer
    if (tid == 0) sm.ntie = 0;
    const int L = load_len(a.len, row / a.Hkv, a.Lmax, a.st, kWhereFinalize);

    pdl_wait();
    pdl_launch_dependents();           // the next kernel may set up; it waits for this one
    // The first round of scores is requested before the item count is known
    // (bounded by the buffer; items past the count are masked below).
    float4 va[kRowU], vb[kRowU];
    auto load_round = [&](float4 (&v)[kRowU], int r, int lim4) {
#pragma unroll
        for (int u = 0; u < kRowU; ++u) {
            const int f = r * kRowRound4 + u * kRowThreads + tid;
            v[u] = f < lim4 ? __ldcg(S4 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    load_round(va, 0, cap4);
    const int n = refine ? min(min(__ldcg(a.src_off + (size_t)row * (src_kappa + 1) + src_kappa), L),
                               min(cap, cstride))
                         : min(L, min(cap, cstride));
    const bool all = n <= a.kappa;
    for (int i = tid; i < kHistBins; i += kRowThreads) {
        sm.hist[i] = all ? 0u : __ldcg(hist_g + i);
        if (!a.keep_hist) hist_g[i] = 0u;              // left zeroed for the next use
    }
    __syncthreads();
    int b1i = 0, above1 = 0;
    if (!all) threshold_bin(sm, kHistBins, a.kappa, &b1i, &above1);
    const uint32_t b1 = (uint32_t)b1i;
    const int need1 = a.kappa - above1;

    // 2. mark the items above the first-digit bin, list those in it
    const int lim4 = (skew + n + 3) >> 2;
    const int nrounds = (lim4 + kRowRound4 - 1) / kRowRound4;
    auto process = [&](const float4 (&v)[kRowU], int r) {
#pragma unroll
        for (int u = 0; u < kRowU; ++u) {
            const int f = r * kRowRound4 + u * kRowThreads + tid;
            const float vals[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t bits = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = 4 * f + q - skew;
                if (i < 0 || i >= n) continue;
                const uint32_t key = score_key(vals[q]);
                const uint32_t d = key >> (32 - kHistBits);
                if (all || d > b1) {
                    bits |= 1u << q;
                } else if (d == b1) {
                    const int e = atomicAdd(&sm.ntie, 1);
                    const uint64_t it = ((uint64_t)key << 32) | (uint32_t)i;
                    if (e < kRowTieCap) ties[e] = it;
                    else tie_g[e] = it;
                }
            }
            // lanes 8w..8w+7 hold the 32 items of bitmap word w of the warp's 128
            uint32_t x = bits << (4 * (lane & 7));
            x |= __shfl_xor_sync(0xffffffffu, x, 1);
            x |= __shfl_xor_sync(0xffffffffu, x, 2);
            x |= __shfl_xor_sync(0xffffffffu, x, 4);
            if ((lane & 7) == 0) bm[(f - lane) / 8 + lane / 8] = x;
        }
    };
    for (int r = 0; r < nrounds; r += 2) {
        if (r + 1 < nrounds) load_round(vb, r + 1, lim4);
        process(va, r);
        if (r + 1 < nrounds) {
            if (r + 2 < nrounds) load_round(va, r + 2, lim4);
            process(vb, r + 1);
        }
    }
    __syncthreads();

    // 3. the exact kappa-th key among the ties; mark the selected ties
    const int m = sm.ntie;
    auto tie_at = [&](int e) -> uint64_t { return e < kRowTieCap ? ties[e] : __ldcg(tie_g + e); };
    auto mark = [&](uint64_t it) {
        const int v = (int)(uint32_t)it + skew;
        atomicOr(&bm[v >> 5], 1u << (v & 31));
    };
    if (!all) mark_selected_ties(sm, tie_at, mark, m, b1, need1);
    __syncthreads();

    // 4. the marked items in index order
    const int W = (skew + n + 31) >> 5;
    const int per = (W + kRowThreads - 1) / kRowThreads;
    const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
    int total;
    int o = block_exclusive_scan(cnt, sm.scratch, &total);
    const int kap = a.kappa;
    for (int w = w0; w < w1; ++w) {
        uint32_t x = bm[w];
        while (x) {
            const int b = __ffs(x) - 1;
            x &= x - 1;
            if (o < kap) sel[o] = 32 * w + b - skew;
            ++o;
        }
    }
    __syncthreads();
    const int nsel = min(total, kap);
    if (refine) {
        for (int j0 = 0; j0 < nsel; j0 += 4 * kRowThreads) {
            int p[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * kRowThreads + tid;
                p[u] = j < nsel ? __ldcg(cpos + sel[j]) : -1;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * kRowThreads + tid;
                if (j < nsel) sel[j] = p[u];
            }
        }
    }
    for (int j = tid; j < kap; j += kRowThreads) {
        if (j >= nsel) sel[j] = -1;
        out[j] = sel[j];
    }
    if (tid == 0 && total != min(kap, n)) report(a.st, kDevErrInternal, kWhereFinalize, (uint32_t)total);
    if (a.prop_off) {
        __syncthreads();
        proposal_offsets(sel, kap, a.radius, L, a.prop_off + (size_t)row * (kap + 1), sm.scratch, a.st);
    }
}

// ---------------------------------------------------------------------------
// Refined layers: the rescoring kernel leaves a row's candidates as runs of
// (key << 32 | position) items, each run ordered by first radix digit,
// highest first.  One block per row (and per batched layer z):
//   1. the head of every run is fetched (cp.async) together with the run
//      counts and the row's histogram, which gives the first digit b1 of the
//      kappa-th key;
//   2. one warp per run walks it from the top, marks the positions of digit
//      above b1 in a shared-memory bitmap over [0, len) and counts the items
//      of digit b1, stopping at the first item below b1; a second walk,
//      after one barrier, lists those ties at the warp's offset (no atomic
//      round trips) with a histogram of their next 11 bits;
//   3. that histogram gives the second digit of the kappa-th key; the ties
//      above it are marked, and the few in its bin are ranked directly (a
//      crowded bin falls back to a 10-bit histogram and a radix select on the
//      position);
//   4. the bitmap, enumerated word by word (per warp, one barrier for the
//      warps' offsets), is the selection in ascending position order; it is
//      staged in shared memory and written out coalesced.  (Two other
//      enumerations were measured slower: a warp-uniform loop predicated per
//      lane, and a fixed share of outputs per thread found by binary search:
//      both are chains of dependent shared-memory loads.)
// Bin searches are warp-parallel (hardware warp sums, one scan in the warp
// that holds the answer): a block-wide scan costs a few hundred cycles of
// dependent shuffles and barriers, the largest cost of such a kernel.
constexpr int kRunSelThreads = 512;
constexpr int kRunSelWarps = kRunSelThreads / 32;
constexpr int kRunSelMaxFetch = 8192;          // run-head items fetched up front, at most
constexpr int kRunSelMaxFetchRuns = kRunSelMaxFetch / 32;

struct RunShared {
    uint32_t hist[kHistBins];      // first digits; reused by the crowded-bin fallback
    uint32_t hist2[kHistBins];     // next 11 bits of the first-digit ties
    int scratch[2 * kSelMaxWarps + 8];
    int thr[2];
    int wsum[kRunSelWarps];
    int nsum[kRunSelWarps];
    int cnt[kRunSelMaxFetchRuns];  // items of each run (when the heads are fetched)
    int ntie;
    int n_small;
    uint64_t small[kSmallCap];
};

// bitmap words: whole rounds of 32 lanes x 4 words for every warp
__host__ __device__ inline int run_words_per_warp(int Lmax) {
    const int W = (Lmax + 31) >> 5;
    const int per = (W + kRunSelWarps - 1) / kRunSelWarps;
    return (per + 127) & ~127;
}
// Items of every run's head fetched up front (0: none, for very many runs):
// at most kRunSelMaxFetch items (64 KB), half that beside a bitmap of more
// than 64 KB.
__host__ __device__ inline int run_prefetch_items(int nruns, int Lmax) {
    const long long budget = (long long)run_words_per_warp(Lmax) * kRunSelWarps * 4 > 65536
                                 ? kRunSelMaxFetch / 2 : kRunSelMaxFetch;
    int pre = 512;
    while (pre > 32 && (long long)nruns * pre > budget) pre >>= 1;
    return (long long)nruns * pre > budget ? 0 : pre;
}
constexpr int kRunSelStage = 8192;   // selections staged in shared memory up to this size
__host__ __device__ inline size_t run_select_smem(int Lmax, int nruns, int kappa) {
    return (size_t)run_words_per_warp(Lmax) * kRunSelWarps * 4 + (size_t)kRowTieCap * 8 +
           (size_t)nruns * run_prefetch_items(nruns, Lmax) * 8 +
           (kappa <= kRunSelStage ? (size_t)kappa * 4 : 0);
}

__global__ void __launch_bounds__(kRunSelThreads, 1) k_select_runs(RunSelectArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ __align__(16) RunShared sm;
    const int wpw = run_words_per_warp(a.Lmax);
    uint32_t *bm = reinterpret_cast<uint32_t *>(dyn);
    uint64_t *ties = reinterpret_cast<uint64_t *>(dyn + (size_t)wpw * kRunSelWarps * 4);
    uint64_t *pre = ties + kRowTieCap;
    const int npre = run_prefetch_items(a.nruns, a.Lmax);
    int32_t *sel = reinterpret_cast<int32_t *>(pre + (size_t)a.nruns * npre);   // staged selection
    const int row = blockIdx.y;
    const size_t z = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint64_t *runs = a.runs + z * a.zruns + (size_t)row * a.nruns * kRunCap;
    const int32_t *rc = a.run_cnt + z * a.zcnt + (size_t)row * a.nruns;
    uint32_t *hist_g = a.hist + z * a.zhist + (size_t)row * kHistBins;
    uint64_t *tie_g = a.tie_spill + z * a.ztie + (size_t)row * a.tie_cap;
    int32_t *out = (a.nz > 1 ? a.outz[z] : a.idx_out) + (size_t)row * a.kappa;
    const int L = load_len(a.len, row / a.Hkv, a.Lmax, a.st, kWhereFinalize);
    {
        uint4 *b4 = reinterpret_cast<uint4 *>(bm);
        for (int i = tid; i < wpw * kRunSelWarps / 4; i += kRunSelThreads) b4[i] = make_uint4(0, 0, 0, 0);
        uint4 *h4 = reinterpret_cast<uint4 *>(sm.hist2);
        for (int i = tid; i < kHistBins / 4; i += kRunSelThreads) h4[i] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) sm.ntie = 0;

    pdl_wait();
    pdl_launch_dependents();           // the next kernel may set up; it waits for this one
    // 1. run counts, the histogram (left zeroed), the heads of the runs
    int mine = 0;
    for (int r = tid; r < a.nruns; r += kRunSelThreads) {
        const int c = min(max(__ldcg(rc + r), 0), kRunCap);
        if (npre > 0) sm.cnt[r] = c;             // npre > 0: at most kRunSelMaxFetchRuns runs
        mine += c;
    }
    {
        const uint4 *hg4 = reinterpret_cast<const uint4 *>(hist_g);
        uint4 *hs4 = reinterpret_cast<uint4 *>(sm.hist);
        for (int i = tid; i < kHistBins / 4; i += kRunSelThreads) {
            hs4[i] = __ldcg(hg4 + i);
            reinterpret_cast<uint4 *>(hist_g)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    const int pieces = npre / 2;
    for (int q = tid; q < a.nruns * pieces; q += kRunSelThreads) {
        const int r = q / pieces, e = 2 * (q - r * pieces);
        cp_async16(pre + (size_t)r * npre + e, runs + (size_t)r * kRunCap + e, 16u);
    }
    cp_async_commit();
    const int nw = __reduce_add_sync(0xffffffffu, mine);
    if (lane == 0) sm.nsum[warp] = nw;
    cp_async_wait<0>();
    __syncthreads();
    int n = 0;
#pragma unroll
    for (int w = 0; w < kRunSelWarps; ++w) n += sm.nsum[w];
    const bool all = n <= a.kappa;
    int b1i = 0, above1 = 0;
    if (!all) find_bin_2048<kRunSelWarps>(sm.hist, a.kappa, sm.wsum, sm.thr, &b1i, &above1);
    const uint32_t b1 = (uint32_t)b1i;
    const int need1 = a.kappa - above1;

    // 2. the heads of the runs, all at once: thread t takes fetched items t,
    //    t + 512, ... (run f / npre, rank f % npre); a run is ordered by first
    //    digit, so items below b1 just drop out.  One shared atomic a warp
    //    places its ties.
    auto mark = [&](uint64_t it) {
        const int p = (int)(uint32_t)it;
        if (p >= 0 && p < L) atomicOr(&bm[p >> 5], 1u << (p & 31));
    };
    const unsigned lt = (1u << lane) - 1u;
    auto add_tie = [&](uint64_t it, int k) {
        if (k < kRowTieCap) ties[k] = it;
        else if (k < a.tie_cap) tie_g[k] = it;
        atomicAdd(&sm.hist2[((uint32_t)(it >> 32) >> 10) & 0x7ffu], 1u);
    };
    constexpr int kChunks = kRunSelMaxFetch / kRunSelThreads;
    const int nf = a.nruns * npre;                       // a multiple of 32
    const int sh = npre > 0 ? __ffs(npre) - 1 : 0;
    uint32_t tmask[kChunks];
    int wt = 0;
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
        const int f = c * kRunSelThreads + tid;
        bool tie = false;
        if (f < nf && (f & (npre - 1)) < sm.cnt[f >> sh]) {
            const uint64_t it = pre[f];
            const uint32_t d = (uint32_t)(it >> 32) >> (32 - kHistBits);
            if (all || d > b1) mark(it);
            tie = !all && d == b1;
        }
        tmask[c] = __ballot_sync(0xffffffffu, tie);
        wt += __popc(tmask[c]);
    }
    int base = 0;
    if (lane == 0 && wt) base = atomicAdd(&sm.ntie, wt);
    base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
        if ((tmask[c] >> lane) & 1u) add_tie(pre[c * kRunSelThreads + tid], base + __popc(tmask[c] & lt));
        base += __popc(tmask[c]);
    }
    // Runs whose needed head is longer than what was fetched: one warp each,
    // from global memory, until the first item below b1.
    for (int r = warp; r < a.nruns; r += kRunSelWarps) {
        const int cr = min(max(__ldcg(rc + r), 0), kRunCap);
        if (cr <= npre) continue;
        if (npre > 0 && !all) {
            const uint32_t dl = (uint32_t)(pre[(size_t)r * npre + npre - 1] >> 32) >> (32 - kHistBits);
            if (dl < b1) continue;
        }
        for (int e0 = npre; e0 < cr; e0 += 32) {
            const int e = e0 + lane;
            const bool v = e < cr;
            const uint64_t it = v ? __ldcg(runs + (size_t)r * kRunCap + e) : 0ull;
            const uint32_t d = (uint32_t)(it >> 32) >> (32 - kHistBits);
            if (v && (all || d > b1)) mark(it);
            const unsigned tm = __ballot_sync(0xffffffffu, v && !all && d == b1);
            if (tm) {
                int tb = 0;
                if (lane == 0) tb = atomicAdd(&sm.ntie, __popc(tm));
                tb = __shfl_sync(0xffffffffu, tb, 0);
                if ((tm >> lane) & 1u) add_tie(it, tb + __popc(tm & lt));
            }
            if (!all && __any_sync(0xffffffffu, v && d < b1)) break;
        }
    }
    if (tid == 0) sm.n_small = 0;
    __syncthreads();

    // 3. the ties
    const int m = min(sm.ntie, a.tie_cap);
    auto tie_at = [&](int e) -> uint64_t { return e < kRowTieCap ? ties[e] : __ldcg(tie_g + e); };
    if (!all && m > 0) {
        if (need1 >= m) {
            for (int e = tid; e < m; e += kRunSelThreads) mark(tie_at(e));
        } else {
            int b2, above2;
            find_bin_2048<kRunSelWarps>(sm.hist2, need1, sm.wsum, sm.thr, &b2, &above2);
            const int need2 = need1 - above2;
            const uint32_t hi21 = (b1 << 21) | ((uint32_t)b2 << 10);
            if ((int)sm.hist2[b2] <= kSmallCap) {
                for (int e = tid; e < m; e += kRunSelThreads) {
                    const uint64_t it = tie_at(e);
                    const uint32_t k21 = (uint32_t)(it >> 32) & 0xfffffc00u;
                    if (k21 > hi21) mark(it);
                    else if (k21 == hi21) sm.small[atomicAdd(&sm.n_small, 1)] = it;
                }
                __syncthreads();
                // rank = items ahead in (key descending, position ascending)
                const int ns = sm.n_small;
                for (int i = tid; i < ns; i += kRunSelThreads) {
                    const uint64_t u = sm.small[i];
                    const uint32_t ku = (uint32_t)(u >> 32);
                    const uint32_t iu = (uint32_t)u;
                    int rk = 0;
                    for (int j = 0; j < ns; ++j) {
                        const uint64_t w = sm.small[j];
                        const uint32_t kw = (uint32_t)(w >> 32);
                        rk += kw > ku || (kw == ku && (uint32_t)w < iu);
                    }
                    if (rk < need2) mark(u);
                }
            } else {
                uint32_t T;
                int cutoff;
                resolve_threshold(sm, tie_at, m, b1, need1, &T, &cutoff);
                for (int e = tid; e < m; e += kRunSelThreads) {
                    const uint64_t it = tie_at(e);
                    const uint32_t k_ = (uint32_t)(it >> 32);
                    if (k_ > T || (k_ == T && (int)(uint32_t)it <= cutoff)) mark(it);
                }
            }
        }
    }
    __syncthreads();

    // 4. the marked positions in ascending order: warp w owns words
    //    [w * wpw, (w + 1) * wpw), 128 a round (4 consecutive words a lane);
    //    one barrier for the warps' offsets; the selection is staged in
    //    shared memory and written out coalesced
    const int WL = (L + 31) >> 5;
    const int wbeg = warp * wpw;
    const int nround = max(0, min(wpw, WL - wbeg) + 127) / 128;
    int wtot = 0;
    for (int rd = 0; rd < nround; ++rd) {
        const uint4 x = *reinterpret_cast<const uint4 *>(bm + wbeg + 128 * rd + 4 * lane);
        wtot += __reduce_add_sync(0xffffffffu, __popc(x.x) + __popc(x.y) + __popc(x.z) + __popc(x.w));
    }
    if (lane == 0) sm.wsum[warp] = wtot;
    __syncthreads();
    int o = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kRunSelWarps; ++w) {
        const int c = sm.wsum[w];
        o += w < warp ? c : 0;
        total += c;
    }
    const int kap = a.kappa;
    const bool staged = kap <= kRunSelStage;
    int32_t *dst = staged ? sel : out;
    for (int rd = 0; rd < nround && o < kap; ++rd) {
        const int w0 = wbeg + 128 * rd + 4 * lane;
        const uint4 x = *reinterpret_cast<const uint4 *>(bm + w0);
        const int c = __popc(x.x) + __popc(x.y) + __popc(x.z) + __popc(x.w);
        int incl = c;
#pragma unroll
        for (int s2 = 1; s2 < 32; s2 <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, s2);
            if (lane >= s2) incl += y;
        }
        int at = o + incl - c;
        const uint32_t ws[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t bits = ws[i];
            while (bits && at < kap) {
                const int bb = __ffs(bits) - 1;
                bits &= bits - 1;
                dst[at++] = 32 * (w0 + i) + bb;
            }
        }
        o += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (staged) {
        __syncthreads();
        for (int j = tid; j < kap; j += kRunSelThreads) out[j] = j < total ? sel[j] : -1;
    } else {
        for (int j = total + tid; j < kap; j += kRunSelThreads) out[j] = -1;
    }
    if (tid == 0 && total != min(kap, n)) report(a.st, kDevErrInternal, kWhereFinalize, (uint32_t)total);
}

cudaError_t launch_select_runs(const RunSelectArgs &a, cudaStream_t s) {
    if (a.nruns < 1) return cudaErrorInvalidValue;
    const size_t smem = run_select_smem(a.Lmax, a.nruns, a.kappa);
    cudaError_t e = cudaFuncSetAttribute(k_select_runs, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int rows = a.B * a.Hkv;
    return launch_kernel(k_select_runs, dim3(1, rows, a.nz > 1 ? a.nz : 1), dim3(kRunSelThreads),
                         smem, s, a);
}

// Whether a selection of `kappa` from rows of at most `items` items runs as
// one block per row, and its dynamic shared memory.
bool select_row_fits(int items, int kappa) {
    return items <= kRowMaxItems && kappa <= kRowMaxKappa;
}

cudaError_t launch_select_row(const SelectArgs &a0, int items, cudaStream_t s) {
    SelectArgs a = a0;
    a.row_cap = items;
    const size_t smem = row_select_smem(items, a.kappa);
    cudaError_t e = cudaFuncSetAttribute(k_select_row, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int rows = a.B * a.Hkv;
    return launch_kernel(k_select_row, dim3(1, rows, a.nz > 1 ? a.nz : 1), dim3(kRowThreads), smem, s, a);
}

}  // namespace prism
