// select.cu -- exact top-kappa selection (Eq. (2) and Eq. (6) of "Prism
// Attention", section 4.1) by one thread-block cluster per (batch, KV head)
// row.
//
// Items are the anchor layer's scores, indexed by position, or a refined
// layer's candidates (score, position), stored contiguously in ascending
// position order by the rescoring kernel.  The C CTAs of a cluster split a
// row's items into C contiguous slices and cooperate through distributed
// shared memory between hardware cluster barriers (no spin-waits, no atomics
// between CTAs).  Scores are compared through order-preserving 32-bit keys
// (equivalently, as floats with -0.0 == +0.0), so every decision is exact:
//   1. each CTA pulls its slice into shared memory with one bulk copy (TMA)
//      per array while its threads read the row's 2048-bin histogram (built
//      by the scoring kernel) and find the first radix digit b1 (the top 11
//      key bits) of the kappa-th score;
//   2. one pass over the slice in shared memory keeps the CTA's candidates --
//      items whose first digit is at least b1, a few percent of the row -- in
//      position order; no other item can be selected.  The ties (first digit
//      == b1) are then picked out of the candidates;
//   3. after one cluster barrier every CTA gathers the ties of all CTAs and
//      resolves the remaining 21 bits on them (an 11-bit and a 10-bit
//      histogram) into the exact kappa-th key T and, if more items equal T
//      than places remain, the cutoff position (a radix select on position).
//      Every CTA computes the same T, so each one knows how many items every
//      CTA selects: its output offset and the last selected position before
//      its slice need no further exchange;
//   4. each CTA writes its selected candidates in order at its offset -- the
//      selection comes out in ascending position order -- and, when asked,
//      the enumeration offsets of the +-r proposal around the new selection,
//      which the next refined layer's rescoring consumes.
#include <cooperative_groups.h>

#include "prism_internal.cuh"

namespace cg = cooperative_groups;

namespace prism {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
// Slice buffer: anchor rows stage up to kChunkScores scores per round; refined
// rows stage kChunkPairs scores and as many positions (second half).  Each
// copy starts up to 12 bytes early (16-byte alignment) and is rounded up to a
// multiple of 16 bytes, hence the slack.  After the pass over the slice the
// buffer holds the gathered ties of the row, then this CTA's selection.
constexpr int kChunkScores = 16384;
constexpr int kChunkPairs = 8192;
constexpr int kHalfBuf = kChunkPairs * 4 + 64;
constexpr int kBufBytes = 2 * kHalfBuf;
constexpr int kTieCache = kBufBytes / 8;         // gathered ties kept in shared memory
constexpr int kSelCache = kBufBytes / 4;         // selected positions kept in shared memory
constexpr int kCandCap = 3072;                   // this CTA's candidates kept in shared memory
constexpr int kMyTieCap = 1024;                  // this CTA's ties kept in shared memory
constexpr int kMaxCluster = 16;
constexpr int kSelDynSmem = kBufBytes + (kCandCap + kMyTieCap) * 8;
static_assert(kChunkScores * 4 + 64 <= kBufBytes, "anchor chunk fits the slice buffer");

struct SelShared {
    uint32_t hist[kHistBins];
    uint64_t bar;                  // completion of the slice copies
    int scratch[2 * kSelWarps + 8];
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
    int warp_cnt[kSelWarps];
    int owned[kMaxCluster];        // proposal positions owned by each CTA's entries
    int fail;
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
    if (lane == 0) sm.warp_cnt[warp] = wcount;
    __syncthreads();
    int res = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kSelWarps; ++w) {
        const int c = sm.warp_cnt[w];
        res += w < warp ? c : 0;
        tot += c;
    }
    __syncthreads();
    *total = tot;
    return res;
}

// The bin of sm.hist[0, nbins) holding the need-th largest item (bins ordered
// by value, the top bin last) and the number of items above it.  All threads;
// contains __syncthreads().
__device__ __forceinline__ void threshold_bin(SelShared &sm, int nbins, int need, int *bin,
                                              int *above) {
    if (threadIdx.x == 0) sm.thr[0] = sm.thr[1] = 0;
    find_threshold_bin(sm.hist, nbins, need, sm.scratch, sm.thr);
    *bin = sm.thr[0];
    *above = sm.thr[1];
    __syncthreads();                               // thr may be reset by the next call
}

__device__ __forceinline__ void zero_hist(SelShared &sm, int nbins) {
    for (int i = threadIdx.x; i < nbins; i += blockDim.x) sm.hist[i] = 0;
    __syncthreads();
}

// Items equal to key T: the index of the rank-th (0-based) lowest, by two
// radix digits of the index (10 + 10 bits; indices < 2^20).  Bins are
// reversed so that the lowest position sits in the top bin.
template <class Get>
__device__ int tie_cutoff(SelShared &sm, Get tie, int m, uint32_t T, int rank) {
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
// (need1 = places left after the items above that bin), and the cutoff index
// among the items equal to T.  All threads.
template <class Get>
__device__ void resolve_threshold(SelShared &sm, Get tie, int m, uint32_t b1, int need1,
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

// Bytes of the 16-byte-aligned span covering [p, p + cnt) 4-byte elements,
// and how many elements precede p in it.
__device__ __forceinline__ uint32_t span_bytes(const void *p, int cnt) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    const uintptr_t a0 = a & ~(uintptr_t)15;
    return cnt > 0 ? (uint32_t)(((a + (uintptr_t)cnt * 4 - a0) + 15) & ~(uintptr_t)15) : 0u;
}
__device__ __forceinline__ int span_skew(const void *p) {
    return (int)((reinterpret_cast<uintptr_t>(p) & 15) >> 2);
}
__device__ __forceinline__ void bulk_span(void *dst, const void *p, int cnt, uint64_t *bar,
                                          uint64_t pol) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p) & ~(uintptr_t)15;
    if (cnt > 0) bulk_load(dst, reinterpret_cast<const void *>(a0), span_bytes(p, cnt), bar, pol);
}

// At most 80 registers a thread, so that a select CTA fits on an SM beside a
// CTA of the anchor scoring kernel running concurrently on another stream.
__global__ void __maxnreg__(80)
k_select(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t dyn[];
    const int32_t *buf_p = reinterpret_cast<const int32_t *>(dyn + kHalfBuf);  // positions (refine)
    uint64_t *tie_all = reinterpret_cast<uint64_t *>(dyn);         // later: the row's ties
    int32_t *sel_s = reinterpret_cast<int32_t *>(dyn);             // later: this CTA's selection
    uint64_t *cand_s = reinterpret_cast<uint64_t *>(dyn + kBufBytes);   // (key << 32 | position)
    uint64_t *mytie = cand_s + kCandCap;
    __shared__ SelShared sm;
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int row = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = (1u << lane) - 1u;
    const int L = load_len(a.len, row / a.Hkv, a.Lmax, a.st, kWhereFinalize);
    if (tid == 0) {
        sm.fail = 0;
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
    }
    const bool refine = a.cpos != nullptr;
    // A refined row's candidate count was written by the selection two
    // kernels back (the rescoring kernel in between waited for it before
    // letting this grid start), so it may be read before the wait.
    const int n = refine ? min(min(__ldcg(a.src_off + (size_t)row * (a.kappa + 1) + a.kappa), L), a.Lmax) : L;
    const float *S = a.S + (size_t)row * a.Lmax;
    const int32_t *cpos = refine ? a.cpos + (size_t)row * a.Lmax : nullptr;
    int32_t *out = a.idx_out + (size_t)row * a.kappa;
    // Overflow areas of the row: candidates beyond kCandCap in the first Lmax
    // entries, ties beyond kMyTieCap in the second, each at the slice's offset.
    uint64_t *spill = a.cspill + (size_t)row * 2 * a.Lmax;
    uint64_t *tie_g = spill + a.Lmax;
    const bool all = n <= a.kappa;
    const int per_cta = (n + C - 1) / C;
    auto slice_begin = [&](int r) { return min(n, r * per_cta); };
    const int i_begin = slice_begin(rank), i_end = min(n, i_begin + per_cta);
    const int chunk = refine ? kChunkPairs : kChunkScores;
    const uint64_t pol = l2_evict_first_policy();
    auto issue_chunk = [&](int c0) {                         // thread 0
        const int cnt = min(chunk, i_end - c0);
        const uint32_t bytes = span_bytes(S + c0, cnt) + (refine ? span_bytes(cpos + c0, cnt) : 0u);
        if (bytes == 0) return;
        mbar_arrive_expect_tx(&sm.bar, bytes);
        bulk_span(dyn, S + c0, cnt, &sm.bar, pol);
        if (refine) bulk_span(dyn + kHalfBuf, cpos + c0, cnt, &sm.bar, pol);
    };
    __syncthreads();                                         // the mbarrier is initialised
    pdl_wait();
    if (tid == 0 && i_begin < i_end) issue_chunk(i_begin);

    // 1. the first digit b1 while the slice is in flight
    int b1i = 0, above1 = 0;
    if (!all) {
        const uint32_t *hg = a.hist + (size_t)row * kHistBins;
        for (int i = tid; i < kHistBins; i += kSelThreads) sm.hist[i] = __ldcg(hg + i);
        __syncthreads();
        threshold_bin(sm, kHistBins, a.kappa, &b1i, &above1);
    }
    const uint32_t b1 = (uint32_t)b1i;
    const int need1 = a.kappa - above1;
    const float f_lo = all ? -INFINITY : digit_floor(b1);   // candidate: s >= f_lo

    // 2. the candidates in position order (4 items a lane per step)
    auto cand_at = [&](int c) -> uint64_t { return c < kCandCap ? cand_s[c] : __ldcg(spill + i_begin + c); };
    int ncand = 0;
    uint32_t phase = 0;
    for (int c0 = i_begin; c0 < i_end; c0 += chunk, phase ^= 1u) {
        const int cnt = min(chunk, i_end - c0);
        const float4 *buf4 = reinterpret_cast<const float4 *>(dyn);
        const int ks = span_skew(S + c0);                 // buffer element q holds item q - ks
        const int kp = refine ? span_skew(cpos + c0) : 0;
        const int g4 = (ks + cnt + 3) >> 2;               // float4 groups in the buffer
        const int gw = (g4 + kSelWarps - 1) / kSelWarps;
        const int w0 = min(g4, warp * gw), w1 = min(g4, w0 + gw);
        if (!mbar_wait(&sm.bar, phase, a.wait_ns) && tid == 0) {
            // The copy never landed: record it and carry on through every
            // cluster barrier (the results of this row are then void).
            report(a.st, kDevErrTimeout, kWhereFinalize, (uint32_t)c0);
            sm.fail = 1;
        }
        auto flags = [&](int g) -> uint32_t {             // candidate bits of group g
            if (g >= w1) return 0u;
            const float4 v = buf4[g];
            const int i0 = 4 * g - ks;
            uint32_t f = 0;
            f |= (uint32_t)(i0 + 0 >= 0 && i0 + 0 < cnt && (all || v.x >= f_lo)) << 0;
            f |= (uint32_t)(i0 + 1 >= 0 && i0 + 1 < cnt && (all || v.y >= f_lo)) << 1;
            f |= (uint32_t)(i0 + 2 >= 0 && i0 + 2 < cnt && (all || v.z >= f_lo)) << 2;
            f |= (uint32_t)(i0 + 3 >= 0 && i0 + 3 < cnt && (all || v.w >= f_lo)) << 3;
            return f;
        };
        int wc = 0;
        for (int g = w0 + lane; g - lane < w1; g += 32) wc += __reduce_add_sync(0xffffffffu, __popc(flags(g)));
        int total;
        int at = ncand + warp_offsets(sm, wc, &total);
        for (int g = w0 + lane; g - lane < w1; g += 32) {
            uint32_t f = flags(g);
            const int cl = __popc(f);
            int incl = cl;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int ci = at + incl - cl;
            if (f) {
                const float *vs = reinterpret_cast<const float *>(buf4 + g);
                while (f) {
                    const int q = __ffs(f) - 1;
                    f &= f - 1;
                    const int i = 4 * g + q - ks;
                    const int p = refine ? buf_p[kp + i] : c0 + i;
                    const uint64_t it = ((uint64_t)score_key(vs[q]) << 32) | (uint32_t)p;
                    if (ci < kCandCap) cand_s[ci] = it;
                    else spill[i_begin + ci] = it;
                    ++ci;
                }
            }
            at += __shfl_sync(0xffffffffu, incl, 31);
        }
        ncand += total;
        __syncthreads();                                  // the buffer is free again
        if (tid == 0 && c0 + chunk < i_end) issue_chunk(c0 + chunk);
    }
    // the ties among the candidates, in order; the last candidate above them
    int ntie = 0, last_sure = -1;
    for (int c0 = 0; c0 < ncand; c0 += kSelThreads) {
        const int c = c0 + tid;
        const uint64_t it = c < ncand ? cand_at(c) : 0;
        const bool t = c < ncand && !all && ((uint32_t)(it >> 32) >> (32 - kHistBits)) == b1;
        if (c < ncand && !t) last_sure = max(last_sure, (int)(uint32_t)it);
        const unsigned mt = __ballot_sync(0xffffffffu, t);
        int round_total;
        const int woff = warp_offsets(sm, __popc(mt), &round_total);
        if (t) {
            const int ti = ntie + woff + __popc(mt & lt);
            if (ti < kMyTieCap) mytie[ti] = it;
            else tie_g[i_begin + ti] = it;
        }
        ntie += round_total;
    }
    for (int o = 16; o >= 1; o >>= 1) last_sure = max(last_sure, __shfl_xor_sync(0xffffffffu, last_sure, o));
    if (lane == 0) sm.scratch[warp] = last_sure;
    __syncthreads();
    if (tid == 0) {
        int ls = -1;
        for (int w = 0; w < kSelWarps; ++w) ls = max(ls, sm.scratch[w]);
        sm.last_sure = ls;
        sm.ntie = ntie;
        sm.nsure = ncand - ntie;
    }
    cluster.sync();     // every CTA's candidates, ties and summary are in place

    // 3. every CTA: all ties of the row -> T, cutoff; its offset and predecessor
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
    const int m = sm.tie_beg[C];
    auto owner = [&](int e) {                     // CTA holding the e-th tie of the row
        int r = 0;
        while (r + 1 < C && sm.tie_beg[r + 1] <= e) ++r;
        return r;
    };
    auto tie_src = [&](int e) -> uint64_t {       // e-th tie of the row, in CTA order
        const int r = owner(e);
        const int t = e - sm.tie_beg[r];
        return t < kMyTieCap ? cluster.map_shared_rank(mytie, r)[t] : __ldcg(tie_g + slice_begin(r) + t);
    };
    const bool local_ok = m <= kTieCache;
    if (local_ok) {
        for (int e = tid; e < m; e += kSelThreads) tie_all[e] = tie_src(e);
        __syncthreads();
    }
    uint32_t T = 0;
    int cutoff = 0x7fffffff;
    if (!all) {
        if (local_ok) resolve_threshold(sm, [&](int e) { return tie_all[e]; }, m, b1, need1, &T, &cutoff);
        else resolve_threshold(sm, tie_src, m, b1, need1, &T, &cutoff);   // very many ties
        // selected ties per CTA, and the last selected tie position per CTA
        for (int e0 = 0; e0 < m; e0 += kSelThreads) {
            const int e = e0 + tid;
            const uint64_t it = e < m ? (local_ok ? tie_all[e] : tie_src(e)) : 0;
            const uint32_t k_ = (uint32_t)(it >> 32);
            const int p = (int)(uint32_t)it;
            const bool f = e < m && (k_ > T || (k_ == T && p <= cutoff));
            const int r = e < m ? owner(e) : -1;
            const unsigned grp = __match_any_sync(0xffffffffu, r) & __ballot_sync(0xffffffffu, f);
            if (f && lane == __ffs(grp) - 1) atomicAdd(&sm.chosen[r], __popc(grp));
            if (f && lane == 31 - __clz(grp)) atomicMax(&sm.last_chosen[r], p);
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

    // 4. write this CTA's selected candidates in order (and keep them)
    int done = base;
    for (int c0 = 0; c0 < ncand; c0 += kSelThreads) {
        const int c = c0 + tid;
        const uint64_t it = c < ncand ? cand_at(c) : 0;
        const uint32_t k_ = (uint32_t)(it >> 32);
        const bool f = c < ncand && (all || k_ > T || (k_ == T && (int)(uint32_t)it <= cutoff));
        const unsigned mk = __ballot_sync(0xffffffffu, f);
        int round_total;
        const int woff = warp_offsets(sm, __popc(mk), &round_total);
        if (f) {
            const int o = done + woff + __popc(mk & lt);
            if (o < a.kappa) out[o] = (int)(uint32_t)it;
            if (o - base < kSelCache) sel_s[o - base] = (int)(uint32_t)it;
        }
        done += round_total;
    }
    if (rank == C - 1) {
        if (tid == 0 && !sm.fail && total != min(a.kappa, n))
            report(a.st, kDevErrInternal, kWhereFinalize, (uint32_t)total);
        for (int e = total + tid; e < a.kappa; e += kSelThreads) out[e] = -1;
    }
    if (rank == 0) {                 // every CTA has read the histogram by now
        uint32_t *hg = a.hist + (size_t)row * kHistBins;
        for (int i = tid; i < kHistBins; i += kSelThreads) hg[i] = 0u;
    }

    // 5. enumeration offsets of the proposal around the new selection
    if (a.prop_off) {
        __syncthreads();                                  // this CTA's selection is written
        const int j0 = min(base, a.kappa), j1 = min(a.kappa, done);
        auto sel = [&](int j) { return j - j0 < kSelCache ? sel_s[j - j0] : out[j]; };
        auto owned = [&](int j) {
            const int i = sel(j);
            const int prev = j == j0 ? prev_last : sel(j - 1);
            long long l = (long long)i - a.radius;
            if (prev >= 0 && (long long)prev + a.radius + 1 > l) l = (long long)prev + a.radius + 1;
            if (l < 0) l = 0;
            long long h = (long long)i + a.radius;
            if (h > L - 1) h = L - 1;
            return h < l ? 0 : (int)(h - l + 1);
        };
        const int per_t = (j1 - j0 + kSelThreads - 1) / kSelThreads;
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
        int32_t *off = a.prop_off + (size_t)row * (a.kappa + 1);
        run += off0;
        for (int j = t0; j < t1; ++j) {
            off[j] = run;
            run += owned(j);
        }
        if (rank == C - 1)                                // entries past the selection own nothing
            for (int j = min(total, a.kappa) + tid; j <= a.kappa; j += kSelThreads) off[j] = all_total;
    } else {
        cluster.sync();     // no CTA leaves while another may still read its shared memory
    }
    pdl_launch_dependents();
}

// CTAs per row: enough that a slice fits one staged chunk (at most 16).
int select_cluster_size(int items, bool refine) {
    const int chunk = refine ? kChunkPairs : kChunkScores;
    int C = 1;
    while (C < kMaxCluster && (items + C - 1) / C > chunk) C *= 2;
    return C;
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s) {
    static bool attr_done[64] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSelDynSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k_select, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    const int rows = a.B * a.Hkv;
    const bool refine = a.cpos != nullptr;
    const long long bound = refine ? (long long)a.kappa * (2LL * a.radius + 1) : (long long)a.Lmax;
    const int items = (int)(bound < a.Lmax ? bound : a.Lmax);
    const int C = select_cluster_size(items, refine);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, rows);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = kSelDynSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = use_pdl() ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k_select, a);
    count_launches(1);
    return e;
}

}  // namespace prism
