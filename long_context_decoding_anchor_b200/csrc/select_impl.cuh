// select_impl.cuh -- the exact top-kappa selection (Eq. (2) and Eq. (6) of
// "Prism Attention", section 4.1): the radix-threshold helpers shared by the
// cluster selection kernel (select.cu) and the one-CTA-per-row selection
// kernel (select_row.cu), and the cluster-wide part of the former.
//
// A row's items are split among the C CTAs of a thread-block cluster in
// contiguous slices, slice r = [r*n/C, (r+1)*n/C).  Before select_finish runs,
// every CTA has found the first radix digit b1 (top 11 key bits) of the
// kappa-th score from the row's histogram and listed its candidates -- the
// items of its slice whose first digit is at least b1, as (key << 32 |
// position) in position order.  select_finish then:
//   1. picks the ties (first digit == b1) out of the candidates;
//   2. after one cluster barrier, gathers the ties of all CTAs through
//      distributed shared memory, histogramming their next 11 bits on the
//      way; the bin b2 holding the kappa-th key usually has a handful of
//      items, which one warp ranks directly (key descending, position
//      ascending) into the exact kappa-th key T and the cutoff position (a
//      crowded bin falls back to a 10-bit histogram and a radix select on
//      position).  Every CTA computes the same T, so each knows how many items
//      every CTA selects: its output offset and the last selected position
//      before its slice need no further exchange;
//   3. writes the CTA's selected candidates in order -- the selection comes
//      out in ascending position order -- and, when asked, the enumeration
//      offsets of the +-r proposal around the new selection.
// Scores are compared through order-preserving 32-bit keys (equivalently as
// floats with -0.0 == +0.0), so every decision is exact.  There are no
// spin-waits and no atomics between CTAs.
#pragma once

#include <cooperative_groups.h>

#include "prism_internal.cuh"

namespace prism {

namespace cg = cooperative_groups;

constexpr int kSelMaxWarps = 32;
constexpr int kMaxCluster = 16;
constexpr int kSmallCap = 128;     // items of the second-level bin ranked directly

struct SelShared {
    uint32_t hist[kHistBins];
    uint64_t bar;                  // completion of a kernel's own copies
    int scratch[2 * kSelMaxWarps + 8];
    int thr[2];
    // this CTA's summary, read by the others
    int ntie;                      // its ties (first digit == b1)
    int nsure;                     // its candidates above the tie bin
    int last_sure;                 // its last candidate position above the tie bin, or -1
    // per CTA of the cluster (every CTA fills these for all of them)
    int tie_beg[kMaxCluster + 1];
    int nsure_of[kMaxCluster];
    int last_sure_of[kMaxCluster];
    int chosen[kMaxCluster];       // ties of CTA r that are selected
    int last_chosen[kMaxCluster];  // last selected tie position of CTA r, or -1
    int warp_cnt[kSelMaxWarps];
    int owned[kMaxCluster];        // proposal positions owned by each CTA's entries
    int fail;
    int n_small;                   // items in the threshold's second-level bin
    uint64_t small[kSmallCap];
    int small_owner[kSmallCap];
};

// Float value of the smallest key whose first digit is d: the inverse of
// score_key on the digit's lower edge.
__device__ __forceinline__ float digit_floor(uint32_t d) {
    if (d <= 3) return -INFINITY;                 // no finite float has a smaller key
    if (d >= 2048) return INFINITY;
    const uint32_t k = d << (32 - kHistBits);
    const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Block-wide exclusive scan of one count per warp (warp-uniform); returns this
// warp's offset and the block total.  Contains __syncthreads().
__device__ __forceinline__ int warp_offsets(SelShared &sm, int wcount, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    if (lane == 0) sm.warp_cnt[warp] = wcount;
    __syncthreads();
    int res = 0, tot = 0;
    for (int w = 0; w < nwarps; ++w) {
        const int c = sm.warp_cnt[w];
        res += w < warp ? c : 0;
        tot += c;
    }
    __syncthreads();
    *total = tot;
    return res;
}

// The bin of sm.hist[0, nbins) holding the need-th largest item (bins ordered
// by value, the top bin last) and the number of items above it.  nbins is a
// multiple of 256; the first 256 threads own nbins / 256 bins each.  All
// threads; contains __syncthreads().
template <class SM>
__device__ __forceinline__ void threshold_bin(SM &sm, int nbins, int need, int *bin, int *above) {
    const int t = threadIdx.x;
    const int per = nbins / 256;
    const int hi = nbins - t * per;                // thread t owns [hi - per, hi): thread 0 the top
    int local = 0;
    if (t < 256)
        for (int i = 1; i <= per; ++i) local += (int)sm.hist[hi - i];
    if (t == 0) sm.thr[0] = sm.thr[1] = 0;
    int total;
    const int ab = block_exclusive_scan(local, sm.scratch, &total);
    if (t < 256 && ab < need && ab + local >= need) {
        int acc = ab;
        for (int i = 1; i <= per; ++i) {
            const int h = (int)sm.hist[hi - i];
            if (acc + h >= need) {
                sm.thr[0] = hi - i;
                sm.thr[1] = acc;
                break;
            }
            acc += h;
        }
    }
    __syncthreads();
    *bin = sm.thr[0];
    *above = sm.thr[1];
    __syncthreads();                               // thr may be reset by the next call
}

template <class SM>
__device__ __forceinline__ void zero_hist(SM &sm, int nbins) {
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) sm.hist[i] = 0;
    __syncthreads();
}

// The bin of h[0, 2048) holding the need-th largest item (bins ordered by
// value, the top bin last) and the number of items above it, by the NW warps
// of the block: lane l of warp w holds the 2048 / (32 NW) bins of descending
// ranks starting at (32w + l) * 2048 / (32 NW); hardware warp sums, then one
// scan in the warp that holds the answer.  wsum holds NW ints, thr two.  A
// block-wide scan costs a few hundred cycles of dependent shuffles and
// barriers; this costs two barriers.  Whole block.
template <int NW>
__device__ __forceinline__ void find_bin_2048(const uint32_t *h, int need, int *wsum, int *thr,
                                              int *bin, int *above) {
    constexpr int BPL = kHistBins / (32 * NW);            // bins a lane, a multiple of 4
    static_assert(BPL >= 4 && BPL % 4 == 0, "whole 16-byte groups of bins a lane");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b0 = kHistBins - BPL * (32 * warp + lane + 1);
    uint32_t c[BPL];                                      // descending: c[0] is bin b0 + BPL - 1
    int ls = 0;
#pragma unroll
    for (int g = 0; g < BPL / 4; ++g) {
        const uint4 v = *reinterpret_cast<const uint4 *>(h + b0 + 4 * g);
        c[BPL - 1 - 4 * g] = v.x;
        c[BPL - 2 - 4 * g] = v.y;
        c[BPL - 3 - 4 * g] = v.z;
        c[BPL - 4 - 4 * g] = v.w;
        ls += (int)(v.x + v.y + v.z + v.w);
    }
    const int ws = __reduce_add_sync(0xffffffffu, ls);
    if (lane == 0) wsum[warp] = ws;
    if (threadIdx.x == 0) thr[0] = thr[1] = 0;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (before < need && before + ws >= need) {
        int incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int ab = before + incl - ls;
        if (ab < need && ab + ls >= need) {
            int acc = ab;
#pragma unroll
            for (int i = 0; i < BPL; ++i) {
                if (acc + (int)c[i] >= need) {
                    thr[0] = b0 + BPL - 1 - i;
                    thr[1] = acc;
                    break;
                }
                acc += (int)c[i];
            }
        }
    }
    __syncthreads();
    *bin = thr[0];
    *above = thr[1];
}

// Items equal to key T: the position of the rank-th (0-based) lowest, by two
// radix digits of the position (10 + 10 bits; positions < 2^20).  Bins are
// reversed so that the lowest position sits in the top bin.
template <class SM, class Get>
__device__ int tie_cutoff(SM &sm, Get tie, int m, uint32_t T, int rank) {
    zero_hist(sm, 1024);
    for (int e = threadIdx.x; e < m; e += blockDim.x) {
        const uint64_t it = tie(e);
        if ((uint32_t)(it >> 32) == T) atomicAdd(&sm.hist[1023 - (((uint32_t)it >> 10) & 1023)], 1u);
    }
    __syncthreads();
    int bin, above;
    threshold_bin(sm, 1024, rank + 1, &bin, &above);
    const uint32_t hd = 1023 - (uint32_t)bin;
    const int rank2 = rank - above;
    zero_hist(sm, 1024);
    for (int e = threadIdx.x; e < m; e += blockDim.x) {
        const uint64_t it = tie(e);
        if ((uint32_t)(it >> 32) == T && (((uint32_t)it >> 10) & 1023) == hd)
            atomicAdd(&sm.hist[1023 - ((uint32_t)it & 1023)], 1u);
    }
    __syncthreads();
    threshold_bin(sm, 1024, rank2 + 1, &bin, &above);
    return (int)((hd << 10) | (1023 - (uint32_t)bin));
}

// The exact kappa-th key T from the items of first digit b1 among the m given
// (need1 = places left after the items above that bin), and the cutoff
// position among the items equal to T.  All threads.
template <class SM, class Get>
__device__ void resolve_threshold(SM &sm, Get tie, int m, uint32_t b1, int need1,
                                  uint32_t *T_out, int *cutoff_out) {
    zero_hist(sm, kHistBins);                        // bits 20..10
    for (int e = threadIdx.x; e < m; e += blockDim.x) {
        const uint32_t key = (uint32_t)(tie(e) >> 32);
        if ((key >> (32 - kHistBits)) == b1) atomicAdd(&sm.hist[(key >> 10) & 0x7ffu], 1u);
    }
    __syncthreads();
    int b2, above;
    threshold_bin(sm, kHistBins, need1, &b2, &above);
    const int need2 = need1 - above;
    const uint32_t hi21 = (b1 << 21) | ((uint32_t)b2 << 10);
    zero_hist(sm, 1024);                             // bits 9..0
    for (int e = threadIdx.x; e < m; e += blockDim.x) {
        const uint32_t key = (uint32_t)(tie(e) >> 32);
        if ((key & 0xfffffc00u) == hi21) atomicAdd(&sm.hist[key & 0x3ffu], 1u);
    }
    __syncthreads();
    int b3;
    threshold_bin(sm, 1024, need2, &b3, &above);
    const int need = need2 - above;
    const int ties = (int)sm.hist[b3];
    const uint32_t T = hi21 | (uint32_t)b3;
    __syncthreads();
    *T_out = T;
    *cutoff_out = ties > need ? tie_cutoff(sm, tie, m, T, need - 1) : 0x7fffffff;
}

// Everything select_finish needs to know about the row and this CTA.
struct SelectCtx {
    int C, rank;
    int n, L, kappa, radius;      // items of the row, its length, budget, proposal radius
    bool all;                     // n <= kappa: every item is selected
    uint32_t b1;                  // first digit of the kappa-th key
    int need1;                    // places left after the items above digit b1
    int i_begin;                  // this CTA's first item (slice offset)
    // shared memory: candidates (cand_cap), this CTA's ties (mytie_cap), the
    // row's gathered ties (tie_cache; may alias sel_s), the CTA's selection
    // (sel_cache ints)
    uint64_t *cand_s, *mytie, *tie_all;
    int32_t *sel_s;
    int cand_cap, mytie_cap, tie_cache, sel_cache;
    // global overflow areas of the row, indexed by item: candidates, ties
    uint64_t *spill, *tie_g;
    int32_t *out;                 // [kappa]
    int32_t *prop_off;            // nullable: [kappa + 1]
    uint32_t *hist_g;             // the row's global histogram, zeroed here once read
    DevStatus *st;
    uint32_t where;
};

__device__ __forceinline__ int slice_begin_of(int r, int n, int C) {
    return (int)((long long)r * n / C);
}

// Steps 1-3 above; ncand candidates are in ctx.cand_s (and ctx.spill beyond
// cand_cap).  Every CTA of the cluster calls it; it ends with a cluster
// barrier, after which no CTA reads another's shared memory.
static __device__ void select_finish(SelShared &sm, cg::cluster_group &cluster, const SelectCtx &x,
                              int ncand) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x;
    const unsigned lt = (1u << lane) - 1u;
    const int C = x.C, rank = x.rank;
    auto cand_at = [&](int c) -> uint64_t {
        return c < x.cand_cap ? x.cand_s[c] : __ldcg(x.spill + x.i_begin + c);
    };

    // 1. the ties among the candidates, in order; the last candidate above them
    int ntie = 0, last_sure = -1;
    for (int c0 = 0; c0 < ncand; c0 += nthreads) {
        const int c = c0 + tid;
        const uint64_t it = c < ncand ? cand_at(c) : 0;
        const bool t = c < ncand && !x.all && ((uint32_t)(it >> 32) >> (32 - kHistBits)) == x.b1;
        if (c < ncand && !t) last_sure = max(last_sure, (int)(uint32_t)it);
        const unsigned mt = __ballot_sync(0xffffffffu, t);
        int round_total;
        const int woff = warp_offsets(sm, __popc(mt), &round_total);
        if (t) {
            const int ti = ntie + woff + __popc(mt & lt);
            if (ti < x.mytie_cap) x.mytie[ti] = it;
            else x.tie_g[x.i_begin + ti] = it;
        }
        ntie += round_total;
    }
    for (int o = 16; o >= 1; o >>= 1) last_sure = max(last_sure, __shfl_xor_sync(0xffffffffu, last_sure, o));
    if (lane == 0) sm.scratch[warp] = last_sure;
    __syncthreads();
    if (tid == 0) {
        int ls = -1;
        for (int w = 0; w < (nthreads >> 5); ++w) ls = max(ls, sm.scratch[w]);
        sm.last_sure = ls;
        sm.ntie = ntie;
        sm.nsure = ncand - ntie;
    }
    for (int i = tid; i < kHistBins; i += nthreads) sm.hist[i] = 0;   // for the ties' next digit
    cluster.sync();     // every CTA's candidates, ties and summary are in place

    // 2. every CTA: all ties of the row -> T, cutoff; its offset and predecessor
    if (warp == 0) {
        int nt = 0;
        if (lane < C) {
            const SelShared *rs = cluster.map_shared_rank(&sm, lane);
            nt = rs->ntie;
            sm.nsure_of[lane] = rs->nsure;
            sm.last_sure_of[lane] = rs->last_sure;
            sm.chosen[lane] = 0;
            sm.last_chosen[lane] = -1;
        }
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane < C) sm.tie_beg[lane] = incl - nt;
        if (lane == C - 1) sm.tie_beg[C] = incl;
    }
    __syncthreads();
    if (rank == 0 && x.hist_g) {     // every CTA has read the row's histogram by now
        for (int i = tid; i < kHistBins; i += nthreads) x.hist_g[i] = 0u;
    }
    const int m = sm.tie_beg[C];
    auto owner = [&](int e) {                     // CTA holding the e-th tie of the row
        int r = 0;
        while (r + 1 < C && sm.tie_beg[r + 1] <= e) ++r;
        return r;
    };
    auto tie_src = [&](int e) -> uint64_t {       // e-th tie of the row, in CTA order
        const int r = owner(e);
        const int t = e - sm.tie_beg[r];
        return t < x.mytie_cap ? cluster.map_shared_rank(x.mytie, r)[t]
                               : __ldcg(x.tie_g + slice_begin_of(r, x.n, C) + t);
    };
    uint32_t T = 0;
    int cutoff = 0x7fffffff;
    if (!x.all) {
        // The ties' next 11 bits are histogrammed while they are gathered
        // (the histogram was zeroed before the cluster barrier).  The first
        // tie_cache ties are kept in shared memory; the rest, if any, are
        // read from their owners again when needed.
        for (int e = tid; e < m; e += nthreads) {
            const uint64_t it = tie_src(e);
            if (e < x.tie_cache) x.tie_all[e] = it;
            atomicAdd(&sm.hist[((uint32_t)(it >> 32) >> 10) & 0x7ffu], 1u);
        }
        if (tid == 0) sm.n_small = 0;
        __syncthreads();
        auto tie_at = [&](int e) -> uint64_t { return e < x.tie_cache ? x.tie_all[e] : tie_src(e); };
        int b2, above2;
        threshold_bin(sm, kHistBins, x.need1, &b2, &above2);
        const int need2 = x.need1 - above2;
        const uint32_t hi21 = (x.b1 << 21) | ((uint32_t)b2 << 10);
        const int in_b2 = (int)sm.hist[b2];
        if (in_b2 <= kSmallCap) {
            // One pass: per CTA, the ties certainly selected (above the bin)
            // and the last of their positions; the few items of the bin are
            // listed and ranked directly by one warp.
            for (int e0 = 0; e0 < m; e0 += nthreads) {
                const int e = e0 + tid;
                const uint64_t it = e < m ? tie_at(e) : 0;
                const uint32_t k21 = (uint32_t)(it >> 32) & 0xfffffc00u;
                const int p = (int)(uint32_t)it;
                const bool f = e < m && k21 > hi21;
                const int r = e < m ? owner(e) : -1;
                const unsigned grp = __match_any_sync(0xffffffffu, r) & __ballot_sync(0xffffffffu, f);
                if (f && lane == __ffs(grp) - 1) atomicAdd(&sm.chosen[r], __popc(grp));
                if (f && lane == 31 - __clz(grp)) atomicMax(&sm.last_chosen[r], p);
                if (e < m && k21 == hi21) {
                    const int slot = atomicAdd(&sm.n_small, 1);
                    sm.small[slot] = it;
                    sm.small_owner[slot] = r;
                }
            }
            __syncthreads();
            if (warp == 0) {
                // rank = items ahead in (key descending, position ascending);
                // the first need2 are selected, the need2-th gives (T, cutoff)
                const int ns = sm.n_small;
                for (int i = lane; i < ns; i += 32) {
                    const uint64_t u = sm.small[i];
                    const uint32_t ku = (uint32_t)(u >> 32);
                    const int pu = (int)(uint32_t)u;
                    int rk = 0;
                    for (int j = 0; j < ns; ++j) {
                        const uint64_t v = sm.small[j];
                        const uint32_t kv = (uint32_t)(v >> 32);
                        rk += kv > ku || (kv == ku && (int)(uint32_t)v < pu);
                    }
                    if (rk < need2) {
                        atomicAdd(&sm.chosen[sm.small_owner[i]], 1);
                        atomicMax(&sm.last_chosen[sm.small_owner[i]], pu);
                    }
                    if (rk == need2 - 1) {
                        sm.thr[0] = (int)ku;
                        sm.thr[1] = pu;
                    }
                }
            }
            __syncthreads();
            T = (uint32_t)sm.thr[0];
            cutoff = sm.thr[1];
        } else {
            // many items share the bin: resolve the remaining bits by histograms
            resolve_threshold(sm, tie_at, m, x.b1, x.need1, &T, &cutoff);
            for (int e0 = 0; e0 < m; e0 += nthreads) {
                const int e = e0 + tid;
                const uint64_t it = e < m ? tie_at(e) : 0;
                const uint32_t k_ = (uint32_t)(it >> 32);
                const int p = (int)(uint32_t)it;
                const bool f = e < m && (k_ > T || (k_ == T && p <= cutoff));
                const int r = e < m ? owner(e) : -1;
                const unsigned grp = __match_any_sync(0xffffffffu, r) & __ballot_sync(0xffffffffu, f);
                if (f && lane == __ffs(grp) - 1) atomicAdd(&sm.chosen[r], __popc(grp));
                if (f && lane == 31 - __clz(grp)) atomicMax(&sm.last_chosen[r], p);
            }
        }
    }
    __syncthreads();
    int base = 0, total = 0, prev_last = -1;
    for (int r = 0; r < C; ++r) {
        const int cnt = sm.nsure_of[r] + sm.chosen[r];
        if (r < rank) {
            base += cnt;
            if (cnt > 0) prev_last = max(sm.last_sure_of[r], sm.last_chosen[r]);
        }
        total += cnt;
    }

    // 3. write this CTA's selected candidates in order (and keep them)
    int done = base;
    for (int c0 = 0; c0 < ncand; c0 += nthreads) {
        const int c = c0 + tid;
        const uint64_t it = c < ncand ? cand_at(c) : 0;
        const uint32_t k_ = (uint32_t)(it >> 32);
        const bool f = c < ncand && (x.all || k_ > T || (k_ == T && (int)(uint32_t)it <= cutoff));
        const unsigned mk = __ballot_sync(0xffffffffu, f);
        int round_total;
        const int woff = warp_offsets(sm, __popc(mk), &round_total);
        if (f) {
            const int o = done + woff + __popc(mk & lt);
            if (o < x.kappa) x.out[o] = (int)(uint32_t)it;
            if (o - base < x.sel_cache) x.sel_s[o - base] = (int)(uint32_t)it;
        }
        done += round_total;
    }
    if (rank == C - 1) {
        if (tid == 0 && !sm.fail && total != min(x.kappa, x.n))
            report(x.st, kDevErrInternal, x.where, (uint32_t)total);
        for (int e = total + tid; e < x.kappa; e += nthreads) x.out[e] = -1;
    }

    // enumeration offsets of the proposal around the new selection
    if (x.prop_off) {
        __syncthreads();                                  // this CTA's selection is written
        const int j0 = min(base, x.kappa), j1 = min(x.kappa, done);
        auto sel = [&](int j) { return j - j0 < x.sel_cache ? x.sel_s[j - j0] : x.out[j]; };
        auto owned = [&](int j) {
            const int i = sel(j);
            const int prev = j == j0 ? prev_last : sel(j - 1);
            long long l = (long long)i - x.radius;
            if (prev >= 0 && (long long)prev + x.radius + 1 > l) l = (long long)prev + x.radius + 1;
            if (l < 0) l = 0;
            long long h = (long long)i + x.radius;
            if (h > x.L - 1) h = x.L - 1;
            return h < l ? 0 : (int)(h - l + 1);
        };
        const int per_t = (j1 - j0 + nthreads - 1) / nthreads;
        const int t0 = min(j1, j0 + tid * per_t), t1 = min(j1, t0 + per_t);
        int cnt = 0;
        for (int j = t0; j < t1; ++j) cnt += owned(j);
        int cta_total;
        int run = block_exclusive_scan(cnt, sm.scratch, &cta_total);
        if (tid < C) cluster.map_shared_rank(sm.owned, tid)[rank] = cta_total;
        cluster.sync();
        int off0 = 0, all_total = 0;
        for (int r = 0; r < C; ++r) {
            off0 += r < rank ? sm.owned[r] : 0;
            all_total += sm.owned[r];
        }
        run += off0;
        for (int j = t0; j < t1; ++j) {
            x.prop_off[j] = run;
            run += owned(j);
        }
        if (rank == C - 1)                                // entries past the selection own nothing
            for (int j = min(total, x.kappa) + tid; j <= x.kappa; j += nthreads) x.prop_off[j] = all_total;
    } else {
        cluster.sync();     // no CTA leaves while another may still read its shared memory
    }
}

}  // namespace prism
