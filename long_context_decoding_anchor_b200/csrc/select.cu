// select.cu -- exact top-kappa selection of an anchor layer (Eq. (2) of
// "Prism Attention", section 4.1; also Eq. (6) for the stage entry point), by
// one thread-block cluster per (batch, KV head) row.
//
// Items are the anchor layer's scores, indexed by position, or a refined
// layer's candidates (score, position) stored contiguously in ascending
// position order.  Each CTA of the cluster pulls its slice of the row into
// shared memory with 1-D bulk copies (TMA) while its threads read the row's
// 2048-bin histogram (built by the scoring kernel) and find the first radix
// digit b1 of the kappa-th score; one pass with float4 steps then lists its
// candidates (first digit >= b1) in position order, and select_finish
// (select_impl.cuh) resolves the exact threshold across the cluster and
// writes the selection.
#include <atomic>

#include "select_impl.cuh"

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
constexpr int kSelDynSmem = kBufBytes + (kCandCap + kMyTieCap) * 8;
static_assert(kChunkScores * 4 + 64 <= kBufBytes, "anchor chunk fits the slice buffer");

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
    const size_t z = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = load_len(a.len, row / a.Hkv, a.Lmax, a.st, kWhereFinalize);
    const int cstride = a.cstride > 0 ? a.cstride : a.Lmax;
    if (tid == 0) {
        sm.fail = 0;
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
    }
    const bool refine = a.cpos != nullptr;
    // A refined row's candidate count was written by the selection two
    // kernels back (the rescoring kernel in between waited for it before
    // letting this grid start), so it may be read before the wait.
    const int src_kappa = a.src_kappa > 0 ? a.src_kappa : a.kappa;
    const int n = refine ? min(min(__ldcg(a.src_off + (size_t)row * (src_kappa + 1) + src_kappa), L), a.Lmax) : L;
    const float *S = a.S + z * a.zS + (size_t)row * cstride;
    const int32_t *cpos = refine ? a.cpos + z * a.zS + (size_t)row * cstride : nullptr;
    int32_t *out = (a.nz > 1 ? a.outz[z] : a.idx_out) + (size_t)row * a.kappa;
    // Overflow areas of the row: candidates beyond kCandCap in the first
    // cstride entries, ties beyond kMyTieCap in the second, each at the
    // slice's offset.
    uint64_t *spill = a.cspill + z * a.zspill + (size_t)row * 2 * cstride;
    uint64_t *tie_g = spill + cstride;
    const bool all = n <= a.kappa;
    const int i_begin = slice_begin_of(rank, n, C), i_end = slice_begin_of(rank + 1, n, C);
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
        const uint32_t *hg = a.hist + z * a.zhist + (size_t)row * kHistBins;
        for (int i = tid; i < kHistBins; i += kSelThreads) sm.hist[i] = __ldcg(hg + i);
        __syncthreads();
        threshold_bin(sm, kHistBins, a.kappa, &b1i, &above1);
    }
    const uint32_t b1 = (uint32_t)b1i;
    const int need1 = a.kappa - above1;
    const float f_lo = all ? -INFINITY : digit_floor(b1);   // candidate: s >= f_lo

    // 2. the candidates in position order (4 items a lane per step)
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
    SelectCtx x;
    x.C = C; x.rank = rank; x.n = n; x.L = L; x.kappa = a.kappa; x.radius = a.radius;
    x.all = all; x.b1 = b1; x.need1 = need1; x.i_begin = i_begin;
    x.cand_s = cand_s; x.mytie = mytie; x.tie_all = tie_all; x.sel_s = sel_s;
    x.cand_cap = kCandCap; x.mytie_cap = kMyTieCap; x.tie_cache = kTieCache; x.sel_cache = kSelCache;
    x.spill = spill; x.tie_g = tie_g; x.out = out;
    x.prop_off = a.prop_off ? a.prop_off + (size_t)row * (a.kappa + 1) : nullptr;   // single layer
    // zeroed for the next use even if unread, unless another selection reads it too
    x.hist_g = a.keep_hist ? nullptr : a.hist + z * a.zhist + (size_t)row * kHistBins;
    x.st = a.st; x.where = kWhereFinalize;
    select_finish(sm, cluster, x, ncand);
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
    // per device: the kernel's attributes are set (setting them twice is harmless)
    static std::atomic<bool> attr_done[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    if (dev < 0 || dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSelDynSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k_select, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev].store(true, std::memory_order_release);
    }
    const int rows = a.B * a.Hkv;
    const bool refine = a.cpos != nullptr;
    const long long bound = a.n_bound > 0 ? (long long)a.n_bound
                            : refine ? (long long)a.kappa * (2LL * a.radius + 1) : (long long)a.Lmax;
    const int items = (int)(bound < a.Lmax ? bound : a.Lmax);
    // A refined row (a proposal or a pool, tens of thousands of candidates)
    // is selected by one block: its latency is a few block barriers, where a
    // cluster pays cluster barriers and distributed gathers.
    if (refine && select_row_fits(items, a.kappa)) return launch_select_row(a, items, s);
    const int C = select_cluster_size(items, refine);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, rows, a.nz > 1 ? a.nz : 1);
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
