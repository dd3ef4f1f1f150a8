// select.cu -- exact top-kappa selection (Eq. (2) and Eq. (6) of "Prism
// Attention", section 4.1).
//
// Scores are mapped to order-preserving 32-bit keys and selected by radix
// digits 11 + 11 + 10 bits:
//   1. the first-digit histogram is built by the scoring kernel;
//   2. k_select_collect (many CTAs per row) finds the threshold digit b1 and
//      lists every item above it ("sel", fewer than kappa items) and every item
//      on it ("tie", usually a few thousand);
//   3. k_select_finalize (one CTA per row) resolves the two remaining digits
//      on the tie list only, which gives the exact kappa-th key T, takes the
//      items above T and, of the items equal to T, the ones with the lowest
//      positions, and writes the selection in ascending position order through
//      a shared-memory bitmap.  The result never depends on the order in
//      which atomics landed.
#include "prism_internal.cuh"

namespace prism {

constexpr int kCollectThreads = 256;
constexpr int kCollectChunk = 4096;
constexpr int kFinalizeThreads = 1024;

__device__ __forceinline__ int row_items(const SelectArgs &a, int row, int L) {
    return a.cpos ? a.ctl[row].n_prop : L;
}

__global__ void __launch_bounds__(kCollectThreads)
k_select_collect(SelectArgs a) {
    __shared__ uint32_t hist_s[kHistBins];
    __shared__ int scratch[40];
    __shared__ int thr[2];
    const int row = blockIdx.y;
    const int b = row / a.Hkv;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereCollect);
    const int n = row_items(a, row, L);
    if (n <= a.kappa) return;                 // everything is selected
    const int base = blockIdx.x * kCollectChunk;
    if (base >= n) return;
    const int tid = threadIdx.x, lane = tid & 31;

    const uint32_t *hg = a.hist + (size_t)row * kHistBins;
    for (int i = tid; i < kHistBins; i += kCollectThreads) hist_s[i] = __ldcg(hg + i);
    if (tid == 0) thr[0] = thr[1] = 0;
    __syncthreads();
    find_threshold_bin(hist_s, kHistBins, a.kappa, scratch, thr);
    const uint32_t b1 = (uint32_t)thr[0];

    const float *S = a.S + (size_t)row * a.Lmax;
    const int32_t *cpos = a.cpos ? a.cpos + (size_t)row * a.Lmax : nullptr;
    int32_t *sel = a.sel + (size_t)row * a.kappa;
    uint64_t *tie = a.tie + (size_t)row * a.Lmax;
    const unsigned lt = (1u << lane) - 1u;
    const int end = min(n, base + kCollectChunk);
    for (int i0 = base; i0 < end; i0 += kCollectThreads) {
        const int i = i0 + tid;
        bool is_sel = false, is_tie = false;
        uint32_t key = 0;
        int pos = 0;
        if (i < end) {
            key = score_key(__ldcg(S + i));
            pos = cpos ? __ldcg(cpos + i) : i;
            const uint32_t d1 = key >> (32 - kHistBits);
            is_sel = d1 > b1;
            is_tie = d1 == b1;
        }
        const unsigned ms = __ballot_sync(0xffffffffu, is_sel);
        if (ms) {
            const int leader = __ffs(ms) - 1;
            int at = 0;
            if (lane == leader) at = atomicAdd(&a.ctl[row].n_sel, __popc(ms));
            at = __shfl_sync(0xffffffffu, at, leader);
            const int slot = at + __popc(ms & lt);
            if (is_sel && slot < a.kappa) sel[slot] = pos;
        }
        const unsigned mt = __ballot_sync(0xffffffffu, is_tie);
        if (mt) {
            const int leader = __ffs(mt) - 1;
            int at = 0;
            if (lane == leader) at = atomicAdd(&a.ctl[row].n_tie, __popc(mt));
            at = __shfl_sync(0xffffffffu, at, leader);
            const int slot = at + __popc(mt & lt);
            if (is_tie && slot < a.Lmax) tie[slot] = ((uint64_t)key << 32) | (uint32_t)pos;
        }
    }
}

// Position of the rank-th (0-based) set bit of bitmap[0..words), scanning in
// ascending order.  Contains __syncthreads(); result in *out (all threads).
__device__ void nth_set_bit(const uint32_t *bitmap, int words, int rank, int *scratch,
                            int *out) {
    const int seg = (words + blockDim.x - 1) / blockDim.x;
    const int w_begin = min(words, (int)threadIdx.x * seg), w_end = min(words, w_begin + seg);
    int cnt = 0;
    for (int w = w_begin; w < w_end; ++w) cnt += __popc(bitmap[w]);
    int total;
    int off = block_exclusive_scan(cnt, scratch, &total);
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

__global__ void __launch_bounds__(kFinalizeThreads)
k_select_finalize(SelectArgs a) {
    extern __shared__ uint32_t bitmap[];
    __shared__ uint32_t hist_s[kHistBins];
    __shared__ int scratch[40];
    __shared__ int thr[2];
    __shared__ int cutoff_s;
    const int row = blockIdx.x;
    const int b = row / a.Hkv;
    const int tid = threadIdx.x;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereFinalize);
    const int n = row_items(a, row, L);
    int32_t *out = a.idx_out + (size_t)row * a.kappa;
    const int32_t *cpos = a.cpos ? a.cpos + (size_t)row * a.Lmax : nullptr;

    if (n <= a.kappa) {
        // min(kappa, n) = n: every item is selected (already ascending).
        for (int e = tid; e < a.kappa; e += blockDim.x)
            out[e] = e < n ? (cpos ? __ldcg(cpos + e) : e) : -1;
    } else {
        const uint32_t *hg = a.hist + (size_t)row * kHistBins;
        for (int i = tid; i < kHistBins; i += blockDim.x) hist_s[i] = __ldcg(hg + i);
        if (tid == 0) thr[0] = thr[1] = 0;
        __syncthreads();
        find_threshold_bin(hist_s, kHistBins, a.kappa, scratch, thr);
        const uint32_t b1 = (uint32_t)thr[0] & (kHistBins - 1);
        const int above1 = thr[1];
        const int need1 = a.kappa - above1;
        const int m = min(__ldcg(&a.ctl[row].n_tie), a.Lmax);
        const int nsel_raw = __ldcg(&a.ctl[row].n_sel);
        const int nsel = min(nsel_raw, a.kappa);
        if (tid == 0 && nsel_raw != above1)
            report(a.st, kDevErrInternal, kWhereFinalize, (uint32_t)nsel_raw);
        const uint64_t *tie = a.tie + (size_t)row * a.Lmax;

        // Second digit (bits 20..10) over the tie list.
        for (int i = tid; i < kHistBins; i += blockDim.x) hist_s[i] = 0;
        __syncthreads();
        for (int e = tid; e < m; e += blockDim.x) {
            const uint32_t key = (uint32_t)(__ldcg(tie + e) >> 32);
            atomicAdd(&hist_s[(key >> 10) & 0x7ffu], 1u);
        }
        if (tid == 0) thr[0] = thr[1] = 0;
        __syncthreads();
        find_threshold_bin(hist_s, kHistBins, need1, scratch, thr);
        const uint32_t b2 = (uint32_t)thr[0] & (kHistBins - 1);
        const int need2 = need1 - thr[1];

        // Third digit (bits 9..0).
        for (int i = tid; i < kHistBins; i += blockDim.x) hist_s[i] = 0;
        __syncthreads();
        for (int e = tid; e < m; e += blockDim.x) {
            const uint32_t key = (uint32_t)(__ldcg(tie + e) >> 32);
            if (((key >> 10) & 0x7ffu) == b2) atomicAdd(&hist_s[key & 0x3ffu], 1u);
        }
        if (tid == 0) thr[0] = thr[1] = 0;
        __syncthreads();
        find_threshold_bin(hist_s, 1024, need2, scratch, thr);
        const uint32_t b3 = (uint32_t)thr[0] & 1023u;
        const int need = need2 - thr[1];
        const int ties = (int)hist_s[b3];
        const uint32_t T = (b1 << 21) | (b2 << 10) | b3;

        const int words = (L + 31) >> 5;
        if (tid == 0) cutoff_s = 0x7fffffff;
        if (ties > need) {
            // More items equal T than places left: keep the `need` lowest positions.
            for (int w = tid; w < words; w += blockDim.x) bitmap[w] = 0u;
            __syncthreads();
            for (int e = tid; e < m; e += blockDim.x) {
                const uint64_t it = __ldcg(tie + e);
                if ((uint32_t)(it >> 32) == T) {
                    const int p = (int)(uint32_t)it;
                    atomicOr(&bitmap[p >> 5], 1u << (p & 31));
                }
            }
            __syncthreads();
            nth_set_bit(bitmap, words, need - 1, scratch, &cutoff_s);
        }
        for (int w = tid; w < words; w += blockDim.x) bitmap[w] = 0u;
        __syncthreads();
        const int cutoff = cutoff_s;
        const int32_t *sel = a.sel + (size_t)row * a.kappa;
        for (int e = tid; e < nsel; e += blockDim.x) {
            const int p = __ldcg(sel + e);
            atomicOr(&bitmap[p >> 5], 1u << (p & 31));
        }
        for (int e = tid; e < m; e += blockDim.x) {
            const uint64_t it = __ldcg(tie + e);
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
        int off = block_exclusive_scan(cnt, scratch, &total);
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
    // Leave the row's histogram and counters zeroed for the next layer.
    uint32_t *hg = a.hist + (size_t)row * kHistBins;
    for (int i = tid; i < kHistBins; i += blockDim.x) hg[i] = 0u;
    if (tid == 0) {
        a.ctl[row].n_sel = 0;
        a.ctl[row].n_tie = 0;
    }
}

cudaError_t launch_select(const SelectArgs &a, long long max_items, cudaStream_t s) {
    const int rows = a.B * a.Hkv;
    const long long chunks = (max_items + kCollectChunk - 1) / kCollectChunk;
    if (chunks > 0 && max_items > a.kappa) {
        dim3 grid((unsigned)chunks, (unsigned)rows);
        k_select_collect<<<grid, kCollectThreads, 0, s>>>(a);
        count_launches(1);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int smem = ((a.Lmax + 31) / 32) * 4;
    cudaError_t e = cudaFuncSetAttribute(k_select_finalize,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_select_finalize<<<rows, kFinalizeThreads, smem, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace prism
