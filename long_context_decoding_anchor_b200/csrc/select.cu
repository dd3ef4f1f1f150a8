// select.cu -- exact top-kappa selection (Eq. (2) and Eq. (6) of "Prism
// Attention", section 4.1), one kernel launch per layer.
//
// Scores (fp32, indexed by token position) are mapped to order-preserving
// 32-bit keys and selected by radix digits of 11 + 11 + 10 bits:
//   1. the scoring kernel has already built the first-digit histogram;
//   2. every CTA of k_select finds the threshold digit b1 from it and lists
//      its items above b1 ("sel": fewer than kappa per row in total) and on b1
//      ("tie": usually a few thousand), with one atomic per list per CTA;
//   3. the last CTA of each row to finish (an atomic counter, no waiting)
//      resolves the two remaining digits on the tie list alone, which gives
//      the exact kappa-th key T, keeps every item above T and, of the items
//      equal to T, those with the lowest positions, and writes the selection
//      in ascending position order through a shared-memory bitmap.
// Anchor layers select over positions [0, len); refined layers over the
// proposal P, enumerated from the owned ranges of the source selection.  The
// result never depends on the order in which atomics landed.
#include "prism_internal.cuh"

namespace prism {

constexpr int kSelThreads = 512;
constexpr int kAnchorItems = 16;
constexpr int kAnchorChunk = kSelThreads * kAnchorItems;   // positions per CTA (anchor)
constexpr int kPosCap = 2048;                              // proposal positions per round
constexpr int kTieCache = 4096;                            // tie items staged in shared memory

struct SelShared {
    uint32_t hist[kHistBins];
    int scratch[40];
    int thr[2];
    int base_sel, base_tie, is_last, cutoff;
    int lo[kPropEntries];
    int off[kPropEntries + 1];
    int pos[kPosCap];
};

// Threshold digit b1 of the row (all threads get it).  Contains __syncthreads().
__device__ uint32_t first_digit(const SelectArgs &a, int row, SelShared &sh) {
    const uint32_t *hg = a.hist + (size_t)row * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh.hist[i] = __ldcg(hg + i);
    if (threadIdx.x == 0) sh.thr[0] = sh.thr[1] = 0;
    __syncthreads();
    find_threshold_bin(sh.hist, kHistBins, a.kappa, sh.scratch, sh.thr);
    return (uint32_t)sh.thr[0] & (kHistBins - 1);
}

// Block-aggregated reservation of this thread's `ns` sel items and `nt` tie
// items: one atomic per list per CTA; list offsets land in *so, *to.
// Contains __syncthreads().
__device__ __forceinline__ void reserve(const SelectArgs &a, int row, int ns, int nt,
                                        SelShared &sh, int *so, int *to) {
    int tot;
    const int ex = block_exclusive_scan((ns << 16) | nt, sh.scratch, &tot);
    if (threadIdx.x == 0) {
        sh.base_sel = (tot >> 16) ? atomicAdd(&a.ctl[row].n_sel, tot >> 16) : 0;
        sh.base_tie = (tot & 0xffff) ? atomicAdd(&a.ctl[row].n_tie, tot & 0xffff) : 0;
    }
    __syncthreads();
    *so = sh.base_sel + (ex >> 16);
    *to = sh.base_tie + (ex & 0xffff);
}

// Position of the rank-th (0-based) set bit of bitmap[0..words), in ascending
// order.  Contains __syncthreads(); the result lands in *out.
__device__ void nth_set_bit(const uint32_t *bitmap, int words, int rank, int *scratch,
                            int *out) {
    const int seg = (words + blockDim.x - 1) / blockDim.x;
    const int w_begin = min(words, (int)threadIdx.x * seg), w_end = min(words, w_begin + seg);
    int cnt = 0;
    for (int w = w_begin; w < w_end; ++w) cnt += __popc(bitmap[w]);
    int total;
    const int off = block_exclusive_scan(cnt, scratch, &total);
    if (rank >= off && rank < off + cnt) {
        int r = rank - off;
        for (int w = w_begin; w < w_end; ++w) {
            uint32_t bits = bitmap[w];
            const int c = __popc(bits);
            if (r < c) {
                for (; r > 0; --r) bits &= bits - 1;
                *out = (w << 5) + __ffs(bits) - 1;
                break;
            }
            r -= c;
        }
    }
    __syncthreads();
}

// Selection of one row, by the last CTA of the row.  b1 / above1: the first
// digit and the number of items above it (from first_digit).  `tcache` holds
// kTieCache tie items: the tie list is read from L2 once when it fits.
__device__ void finalize_row(const SelectArgs &a, int row, int L, int n, uint32_t b1,
                             int above1, SelShared &sh, uint32_t *bitmap, uint64_t *tcache) {
    const int tid = threadIdx.x;
    int32_t *out = a.idx_out + (size_t)row * a.kappa;
    if (n <= a.kappa) {
        // min(kappa, n) = n: every item is selected, in ascending order.
        if (!a.src) {
            for (int e = tid; e < a.kappa; e += blockDim.x) out[e] = e < n ? e : -1;
        } else {
            const int32_t *src = a.src + (size_t)row * a.kappa;
            int running = 0;
            for (int jb = 0; jb < a.kappa; jb += blockDim.x) {
                int lo = 0, cnt = 0;
                if (jb + tid < a.kappa)
                    cnt = owned_range(src, jb + tid, a.radius, L, &lo, a.st, kWhereFinalize);
                int tot;
                const int ex = block_exclusive_scan(cnt, sh.scratch, &tot);
                for (int i = 0; i < cnt; ++i) {
                    const int o = running + ex + i;
                    if (o < a.kappa) out[o] = lo + i;
                }
                running += tot;
            }
            for (int e = running + tid; e < a.kappa; e += blockDim.x) out[e] = -1;
        }
        return;
    }
    // The kappa-th key T, digit by digit.
    const int need1 = a.kappa - above1;
    const int nsel_raw = __ldcg(&a.ctl[row].n_sel);
    const int nsel = min(nsel_raw, a.kappa);
    const int m = min(__ldcg(&a.ctl[row].n_tie), a.Lmax);
    if (tid == 0 && nsel_raw != above1)
        report(a.st, kDevErrInternal, kWhereFinalize, (uint32_t)nsel_raw);
    const uint64_t *tie_g = a.tie + (size_t)row * a.Lmax;
    const bool cached = m <= kTieCache;
    if (cached)
        for (int e = tid; e < m; e += blockDim.x) tcache[e] = __ldcg(tie_g + e);
    const uint64_t *tie = cached ? tcache : tie_g;

    for (int i = tid; i < kHistBins; i += blockDim.x) sh.hist[i] = 0;
    if (tid == 0) sh.thr[0] = sh.thr[1] = 0;
    __syncthreads();
    for (int e = tid; e < m; e += blockDim.x) {
        const uint32_t key = (uint32_t)(tie[e] >> 32);
        atomicAdd(&sh.hist[(key >> 10) & 0x7ffu], 1u);
    }
    __syncthreads();
    find_threshold_bin(sh.hist, kHistBins, need1, sh.scratch, sh.thr);
    const uint32_t b2 = (uint32_t)sh.thr[0] & (kHistBins - 1);
    const int need2 = need1 - sh.thr[1];

    for (int i = tid; i < kHistBins; i += blockDim.x) sh.hist[i] = 0;
    if (tid == 0) sh.thr[0] = sh.thr[1] = 0;
    __syncthreads();
    for (int e = tid; e < m; e += blockDim.x) {
        const uint32_t key = (uint32_t)(tie[e] >> 32);
        if (((key >> 10) & 0x7ffu) == b2) atomicAdd(&sh.hist[key & 0x3ffu], 1u);
    }
    __syncthreads();
    find_threshold_bin(sh.hist, 1024, need2, sh.scratch, sh.thr);
    const uint32_t b3 = (uint32_t)sh.thr[0] & 1023u;
    const int need = need2 - sh.thr[1];
    const int ties = (int)sh.hist[b3];
    const uint32_t T = (b1 << 21) | (b2 << 10) | b3;

    const int words = (L + 31) >> 5;
    if (tid == 0) sh.cutoff = 0x7fffffff;
    if (ties > need) {
        // More items equal T than places left: keep the `need` lowest positions.
        for (int w = tid; w < words; w += blockDim.x) bitmap[w] = 0u;
        __syncthreads();
        for (int e = tid; e < m; e += blockDim.x) {
            const uint64_t it = tie[e];
            if ((uint32_t)(it >> 32) == T) {
                const int p = (int)(uint32_t)it;
                atomicOr(&bitmap[p >> 5], 1u << (p & 31));
            }
        }
        __syncthreads();
        nth_set_bit(bitmap, words, need - 1, sh.scratch, &sh.cutoff);
    }
    for (int w = tid; w < words; w += blockDim.x) bitmap[w] = 0u;
    __syncthreads();
    const int cutoff = sh.cutoff;
    const int32_t *sel = a.sel + (size_t)row * a.kappa;
    for (int e = tid; e < nsel; e += blockDim.x) {
        const int p = __ldcg(sel + e);
        atomicOr(&bitmap[p >> 5], 1u << (p & 31));
    }
    for (int e = tid; e < m; e += blockDim.x) {
        const uint64_t it = tie[e];
        const uint32_t key = (uint32_t)(it >> 32);
        const int p = (int)(uint32_t)it;
        if (key > T || (key == T && p <= cutoff)) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
    }
    __syncthreads();
    const int seg = (words + blockDim.x - 1) / blockDim.x;
    const int w_begin = min(words, tid * seg), w_end = min(words, w_begin + seg);
    int cnt = 0;
    for (int w = w_begin; w < w_end; ++w) cnt += __popc(bitmap[w]);
    int total;
    int off = block_exclusive_scan(cnt, sh.scratch, &total);
    for (int w = w_begin; w < w_end && off < a.kappa; ++w) {
        uint32_t bits = bitmap[w];
        while (bits && off < a.kappa) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1;
            out[off++] = (w << 5) + bpos;
        }
    }
    if (tid == 0 && total != a.kappa) report(a.st, kDevErrInternal, kWhereFinalize, (uint32_t)total);
    for (int e = total + tid; e < a.kappa; e += blockDim.x) out[e] = -1;
}

__global__ void __launch_bounds__(kSelThreads)
k_select(SelectArgs a) {
    extern __shared__ uint32_t bitmap[];
    __shared__ SelShared sh;
    const int row = blockIdx.y;
    const int b = row / a.Hkv;
    const int tid = threadIdx.x;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereCollect);
    const int n = a.src ? __ldcg(&a.ctl[row].n_prop) : L;
    const float *S = a.S + (size_t)row * a.Lmax;
    int32_t *sel = a.sel + (size_t)row * a.kappa;
    uint64_t *tie = a.tie + (size_t)row * a.Lmax;

    uint32_t b1 = 0;
    int above1 = 0;
    if (n > a.kappa) {
        b1 = first_digit(a, row, sh);
        above1 = sh.thr[1];
        if (!a.src) {
            // Anchor: positions [blockIdx.x * chunk, +chunk).
            const int base = blockIdx.x * kAnchorChunk;
            if (base < n) {
                uint32_t key[kAnchorItems];
                int ns = 0, nt = 0;
#pragma unroll
                for (int k = 0; k < kAnchorItems; ++k) {
                    const int i = base + k * kSelThreads + tid;
                    key[k] = 0;
                    if (i < n) {
                        key[k] = score_key(__ldcg(S + i));
                        const uint32_t d1 = key[k] >> (32 - kHistBits);
                        ns += d1 > b1;
                        nt += d1 == b1;
                    }
                }
                int so, to;
                reserve(a, row, ns, nt, sh, &so, &to);
#pragma unroll
                for (int k = 0; k < kAnchorItems; ++k) {
                    const int i = base + k * kSelThreads + tid;
                    if (i < n) {
                        const uint32_t d1 = key[k] >> (32 - kHistBits);
                        if (d1 > b1) {
                            if (so < a.kappa) sel[so] = i;
                            ++so;
                        } else if (d1 == b1) {
                            if (to < a.Lmax) tie[to] = ((uint64_t)key[k] << 32) | (uint32_t)i;
                            ++to;
                        }
                    }
                }
            }
        } else {
            // Refined layer: the proposal positions owned by 64 source entries.
            const int j0 = blockIdx.x * kPropEntries;
            const int32_t *src = a.src + (size_t)row * a.kappa;
            const int total = proposal_slice(src, j0, a.kappa, a.radius, L, sh.lo, sh.off,
                                             sh.scratch, a.st, kWhereCollect);
            if (total > 0) {
                for (int e0 = 0; e0 < total; e0 += kPosCap) {
                    const int nr = min(kPosCap, total - e0);
                    for (int i = tid; i < nr; i += kSelThreads)
                        sh.pos[i] = slice_position(sh.lo, sh.off, e0 + i);
                    __syncthreads();
                    constexpr int kPer = kPosCap / kSelThreads;
                    uint32_t key[kPer];
                    int ns = 0, nt = 0;
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        const int i = k * kSelThreads + tid;
                        key[k] = 0;
                        if (i < nr) {
                            key[k] = score_key(__ldcg(S + sh.pos[i]));
                            const uint32_t d1 = key[k] >> (32 - kHistBits);
                            ns += d1 > b1;
                            nt += d1 == b1;
                        }
                    }
                    int so, to;
                    reserve(a, row, ns, nt, sh, &so, &to);
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        const int i = k * kSelThreads + tid;
                        if (i < nr) {
                            const uint32_t d1 = key[k] >> (32 - kHistBits);
                            const int p = sh.pos[i];
                            if (d1 > b1) {
                                if (so < a.kappa) sel[so] = p;
                                ++so;
                            } else if (d1 == b1) {
                                if (to < a.Lmax) tie[to] = ((uint64_t)key[k] << 32) | (uint32_t)p;
                                ++to;
                            }
                        }
                    }
                    __syncthreads();
                }
            }
        }
    }

    // The last CTA of the row to get here finalizes it.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(&a.ctl[row].done_select, 1u);
        sh.is_last = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!sh.is_last) return;
    __threadfence();
    const int bitmap_words = (a.Lmax + 31) / 32;
    uint64_t *tcache = reinterpret_cast<uint64_t *>(bitmap + ((bitmap_words + 1) & ~1));
    finalize_row(a, row, L, n, b1, above1, sh, bitmap, tcache);
    // Leave the row's histogram and counters zeroed for the next layer.
    uint32_t *hg = a.hist + (size_t)row * kHistBins;
    for (int i = tid; i < kHistBins; i += blockDim.x) hg[i] = 0u;
    if (tid == 0) {
        a.ctl[row].n_sel = 0;
        a.ctl[row].n_tie = 0;
        a.ctl[row].n_prop = 0;
        a.ctl[row].done_select = 0;
    }
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t s) {
    const int rows = a.B * a.Hkv;
    const int chunks = a.src ? (a.kappa + kPropEntries - 1) / kPropEntries
                             : (a.Lmax + kAnchorChunk - 1) / kAnchorChunk;
    const int words = (a.Lmax + 31) / 32;
    const int smem = ((words + 1) & ~1) * 4 + kTieCache * 8;
    cudaError_t e = cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_select<<<dim3(chunks, rows), kSelThreads, smem, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace prism
