// score.cu -- relevance scoring of the Prism Attention decode step.
//
// Eq. (1) of "Prism Attention" (section 4.1) in the GQA-summed form
//   s(i) = scale * sum_{j in G(h)} <q_j, k_i> = scale * <qbar, k_i>,
//   qbar = sum_{j in G(h)} q_j   (exact re-association, done once per row),
// so every key element costs one FMA: the kernels are bound by HBM bandwidth,
// not by arithmetic, and use CUDA cores, not tensor cores.
//
// k_anchor_score streams the whole key cache of the anchor layer: a
// persistent grid (one CTA per SM) walks a contiguous range of 128-token
// tiles; one producer thread moves each tile (contiguous in memory) into a
// 3-stage shared-memory ring with a 1-D bulk copy (TMA, cp.async.bulk) that
// completes on an mbarrier, and eight consumer warps form the dot products
// from shared memory.  Scores go to global memory (they stay L2-resident for
// the selection) and their top 11 key bits into a per-row histogram, the
// first radix digit of the top-kappa selection.
//
// k_refine_rescore scores only the proposal positions of a refined layer
// (Eq. (5)), enumerated from the owned ranges of the source selection and
// gathered with 16-byte cp.async pieces; the (score, position) candidates
// are stored contiguously at their enumeration index.
#include "prism_internal.cuh"
#include "q2_impl.cuh"
#include "select_impl.cuh"
#include "tiles.cuh"

namespace prism {

template <int D>
struct AnchorCfg {
    static constexpr int kTileRows = 128;
    static constexpr int kStages = 3;
    static constexpr int kConsumerWarps = 8;
    static constexpr int kThreads = 32 * (kConsumerWarps + 1);
    static constexpr int kNL = D / 8;                     // lanes per key row (16 B each)
    static constexpr int kRPI = 32 / kNL;                 // key rows per warp instruction
    static constexpr int kRowsPerWarp = kTileRows / kConsumerWarps;
    static constexpr int kSteps = kRowsPerWarp / kRPI;    // partial sums per lane per tile
    static constexpr int kTileBytes = kTileRows * D * 2;
    static constexpr int kSmemBytes = kStages * kTileBytes + 2 * kStages * 8 + kHistBins * 4 + 64 * 4;
};

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(AnchorCfg<D>::kThreads, 1)
k_anchor_score(ScoreArgs a) {
    using C = AnchorCfg<D>;
    constexpr int TILE = C::kTileRows;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kStages * C::kTileBytes);
    uint64_t *empty = full + C::kStages;
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(empty + C::kStages);
    int *scratch = reinterpret_cast<int *>(hist_s + kHistBins);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int i = tid; i < kHistBins; i += blockDim.x) hist_s[i] = 0;
    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // This CTA's contiguous share of the tile order.
    long long total;
    TileCursor cur0;
    {
        // total is needed before the start tile is known: first pass with t = 0.
        TileCursor dummy;
        locate_tile<TILE>(a.len, a.B, a.Hkv, a.Lmax, 0, &dummy, &total, scratch, a.st);
    }
    const long long t_begin = total * blockIdx.x / gridDim.x;
    const long long t_end = total * (blockIdx.x + 1) / gridDim.x;
    if (t_begin >= t_end) {
        pdl_wait();
        return;
    }
    {
        long long tot2;
        locate_tile<TILE>(a.len, a.B, a.Hkv, a.Lmax, t_begin, &cur0, &tot2, scratch, a.st);
    }
    const int ntiles = (int)(t_end - t_begin);
    if (ntiles <= 0) {
        pdl_wait();
        return;
    }

    if (warp == C::kConsumerWarps) {
        // ---------------- producer: one thread issues the bulk copies -------------
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            const uint16_t *kb = static_cast<const uint16_t *>(a.k);
            TileCursor c = cur0;
            bool failed = false;
            int issued = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!failed && !mbar_wait(&empty[s], ph ^ 1u, a.wait_ns)) {
                    report(a.st, kDevErrTimeout, kWhereScore, (uint32_t)it);
                    failed = true;
                }
                if (!failed) {
                    int L = __ldg(a.len + c.b);
                    L = L < 0 ? 0 : (L > a.Lmax ? a.Lmax : L);
                    const int rows = min(TILE, L - c.j * TILE);
                    const uint32_t bytes = (uint32_t)rows * D * 2;
                    const size_t off = ((size_t)(c.b * a.Hkv + c.h) * a.Lmax + (size_t)c.j * TILE) * D;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_load(stages + s * C::kTileBytes, kb + off, bytes, &full[s], pol);
                    issued = it + 1;
                }
                next_tile<TILE>(c, a.len, a.B, a.Hkv, a.Lmax);
            }
            // Drain: every issued copy must land before the CTA may exit.
            for (int it = max(0, issued - C::kStages); it < issued; ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!mbar_wait(&full[s], ph, a.wait_ns)) {
                    report(a.st, kDevErrTimeout, kWhereScore, 0x80000000u | (uint32_t)it);
                }
            }
        }
        return;
    }

    // ---------------- consumers ------------------------------------------------
    // The key cache is an input: the producer streams it at once.  Scores and
    // the histogram are written only after the preceding kernel has finished.
    pdl_wait();
    const int slice = lane % C::kNL;            // which 8 elements of a key row
    const int sub = lane / C::kNL;              // which row of an instruction's rows
    const int row0 = warp * C::kRowsPerWarp;
    float qreg[8];
    int cur_row = -1;
    TileCursor c = cur0;
    bool failed = false;
    const uint16_t *qb = static_cast<const uint16_t *>(a.q);
    const int Hq = a.Hkv * a.G;

    for (int it = 0; it < ntiles; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
        const int row = c.b * a.Hkv + c.h;
        if (row != cur_row) {
            if (cur_row >= 0) {
                consumer_sync();
                for (int i = tid; i < kHistBins; i += 32 * C::kConsumerWarps) {
                    uint32_t v = hist_s[i];
                    if (v) {
                        atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
                        hist_s[i] = 0;
                    }
                }
                consumer_sync();
            }
            // qbar: sum of the group's query heads, this lane's 8 elements.
#pragma unroll
            for (int e = 0; e < 8; ++e) qreg[e] = 0.f;
            for (int g = 0; g < a.G; ++g) {
                const uint4 w = *reinterpret_cast<const uint4 *>(
                    qb + ((size_t)c.b * Hq + (size_t)c.h * a.G + g) * D + slice * 8);
                qreg[0] += bf16_lo(w.x); qreg[1] += bf16_hi(w.x);
                qreg[2] += bf16_lo(w.y); qreg[3] += bf16_hi(w.y);
                qreg[4] += bf16_lo(w.z); qreg[5] += bf16_hi(w.z);
                qreg[6] += bf16_lo(w.w); qreg[7] += bf16_hi(w.w);
            }
            cur_row = row;
        }
        int L = __ldg(a.len + c.b);
        L = L < 0 ? 0 : (L > a.Lmax ? a.Lmax : L);

        if (!failed && !mbar_wait(&full[s], ph, a.wait_ns)) {
            report(a.st, kDevErrTimeout, kWhereScore, 0x40000000u | (uint32_t)it);
            failed = true;
        }
        if (!failed) {
            const uint8_t *tile = stages + s * C::kTileBytes;
            float part[C::kSteps];
#pragma unroll
            for (int st = 0; st < C::kSteps; ++st) {
                const int r = row0 + st * C::kRPI + sub;
                const uint4 kv = *reinterpret_cast<const uint4 *>(tile + r * (D * 2) + slice * 16);
                part[st] = dot8(kv, qreg);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            transpose_reduce<C::kSteps, C::kNL>(part, lane);
            const int item = transpose_item<C::kSteps, C::kNL>(lane);
            const int pos = c.j * TILE + row0 + item * C::kRPI + sub;
            if (transpose_writer<C::kSteps, C::kNL>(lane) && pos < L) {
                const float sc = part[0] * a.scale;
                a.S[(size_t)row * a.Lmax + pos] = sc;
                atomicAdd(&hist_s[score_key(sc) >> (32 - kHistBits)], 1u);
            }
        }
        next_tile<TILE>(c, a.len, a.B, a.Hkv, a.Lmax);
    }
    consumer_sync();
    // The dependent (the selection) may start only now: launched earlier, its
    // CTAs would sit on SMs for the whole scan, waiting.
    pdl_launch_dependents();
    if (cur_row >= 0) {
        for (int i = tid; i < kHistBins; i += 32 * C::kConsumerWarps) {
            uint32_t v = hist_s[i];
            if (v) atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
        }
    }
}

// ---------------------------------------------------------------------------
// Refined layer: score only the proposal positions (Eq. (5)), and hand the
// selection (Eq. (6)) its candidates already ordered by first radix digit.
//
// The source selection is canonical (ascending, distinct, -1 padded), so the
// proposal -- every position within r of a source entry, clipped to [0, L) --
// splits into the owned ranges of consecutive entries (owned_range): entry j
// owns the positions of its window that no earlier window covers.  Part p of
// a row (blockIdx.x) takes the entries [p*E/P, (p+1)*E/P), counts their
// ranges with one block scan, and lists the positions they own ("slots",
// ascending) in a shared-memory table, one run of kRunCap slots at a time.
// Each warp owns 16 slots of every window of 128 and gathers exactly the
// 16-byte pieces of those key rows that its lanes will read (cp.async, a
// kStages pipeline per warp, no hand-off between warps).  (One 1-D bulk copy
// per 256-byte row was measured slower: the copy engine's rate for small
// copies, not DRAM, then sets the pace.)
// The scores' order-preserving keys go into the table beside the positions;
// at the end of the run the block sorts the (key, position) items by first
// radix digit (a counting sort on its own histogram, which it also adds to
// the row's) and writes them out as one run, highest digit first.  The
// selection then reads only the head of each run.
// Key formats of the rescoring kernel: bf16 keys with the group sum
// (Eq. (1)), bf16 keys with the group maximum (Eq. (9)), 2-bit keys with the
// group maximum (Eq. (7)-(9), row format of q2_impl.cuh).
enum : int { kFmtSum = 0, kFmtMax = 1, kFmtQ2 = 2 };

// ST: windows in a warp's gather pipeline.  Three keep more bytes in
// flight; two (an 89 KB CTA at d = 128) let a rescoring CTA share an SM with
// an anchor-scan CTA and an attention CTA, which a layer whose rows' blocks
// wait for one another needs while anchor scans are in flight.
template <int D, int FMT = kFmtSum, int ST = 3>
struct RescoreCfg {
    static constexpr int kTileRows = 128;              // slots of a window
    static constexpr int kStages = ST;                 // windows in a warp's pipeline
    static constexpr int kWarps = 8;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kRowBytes = FMT == kFmtQ2 ? q2_row_bytes(D) : D * 2;
    // rows read by ldmatrix are padded by 16 bytes: eight consecutive rows
    // then start in eight different bank quads (conflict-free, no swizzle)
    static constexpr int kRowStride = FMT == kFmtMax ? kRowBytes + 16 : kRowBytes;
    static constexpr int kNL = kRowBytes / 16;         // lanes (16-byte pieces) per key row
    static constexpr int kRPI = 32 / kNL;
    static constexpr int kRowsPerWarp = kTileRows / kWarps;   // 16
    static constexpr int kSteps = kRowsPerWarp / kRPI;
    static constexpr int kWarpStage = kRowsPerWarp * kRowStride;
    static constexpr int kStageBytes = kStages * kWarps * kWarpStage;
    static constexpr int kItemOff = kStageBytes;                   // u64 [kRunCap]: key << 32 | position
    static constexpr int kHistOff = kItemOff + kRunCap * 8;
    static constexpr int kScratchOff = kHistOff + kHistBins * 4;
    static constexpr int kSmemBytes = kScratchOff + 48 * 4;
    // each run is sorted in the (then idle) stages
    static constexpr bool kStageSort = kStageBytes >= kRunCap * 8;
    static_assert(kMaxPartEntries % kThreads == 0, "entries split evenly over the threads");
};

// Group maximum (Eq. (9) form) of a warp's 16 gathered rows: the [16 x d] x
// [d x 8] products of mma.sync m16n8k16 (bf16 in, fp32 accumulate; one or two
// n-tiles of 8 heads), A fragments by ldmatrix from rows RS bytes apart
// (conflict-free: rows padded to D*2 + 16 bytes, or rows of D*2 bytes whose
// 16-byte chunk c sits at chunk c ^ (row % 8)), B fragments (the group's
// queries, head n % G in column n) held in registers.  Returns the maxima of
// rows lane/4 (.x) and lane/4 + 8 (.y) of the warp's block, in every lane of
// the quad.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                            uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
template <int D, int RS>
__device__ __forceinline__ float2 group_max_16rows(const uint8_t *rows16, const uint32_t (&qf)[2][D / 16][2],
                                                   bool two_tiles, int lane) {
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
    const int r = (lane & 7) + ((lane >> 3) & 1) * 8;       // row this lane addresses
    const uint32_t base = smem_addr(rows16 + r * RS);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int chunk = 2 * kk + (lane >> 4);
        // rows of D*2 bytes are swizzled (chunk c at c ^ (row % 8)); padded rows are not
        const int at = RS == D * 2 ? (chunk ^ (lane & 7)) : chunk;
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(base + (uint32_t)(at << 4), a0, a1, a2, a3);
        mma_bf16_16816(c0, a0, a1, a2, a3, qf[0][kk][0], qf[0][kk][1]);
        if (two_tiles) mma_bf16_16816(c1, a0, a1, a2, a3, qf[1][kk][0], qf[1][kk][1]);
    }
    float lo = fmaxf(c0[0], c0[1]), hi = fmaxf(c0[2], c0[3]);
    if (two_tiles) {
        lo = fmaxf(lo, fmaxf(c1[0], c1[1]));
        hi = fmaxf(hi, fmaxf(c1[2], c1[3]));
    }
    lo = fmaxf(lo, __shfl_xor_sync(0xffffffffu, lo, 1));
    lo = fmaxf(lo, __shfl_xor_sync(0xffffffffu, lo, 2));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 1));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 2));
    return make_float2(lo, hi);
}

// ---------------------------------------------------------------------------
// Fused selection of a refined layer (Eq. (6)): the blocks of a row, resident
// together, each holding its part's candidates (key << 32 | position, in
// ascending position order) in shared memory.
//   1. every block adds its histogram to the row's; barrier;
//   2. every block reads the row's histogram (the first digit b1 of the
//      kappa-th key), counts its candidates above b1 and publishes its ties
//      (first digit b1) and both counts; barrier;
//   3. every block gathers all ties of the row and resolves the exact kappa-th
//      key T and the cutoff position among the items equal to T (the next 11
//      bits; a handful of items in that bin ranked directly, a crowded bin by
//      histograms); then every part's selected count, hence its offset;
//   4. every block writes its selected positions, in order, at its offset:
//      parts hold ascending disjoint position ranges, so the selection comes
//      out in ascending order.
// The block scans here are warp scans joined by one barrier.
struct EpiView {              // the shared-memory view the threshold helpers take
    uint32_t *hist;
    int *scratch;
    int *thr;
};

// Exclusive prefix of x over the block (NW warps); wsum holds NW ints and is
// free again after the next barrier.  One barrier.
template <int NW>
__device__ __forceinline__ int block_excl_scan_fast(int x, int *wsum, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int v = wsum[w];
        before += w < warp ? v : 0;
        tot += v;
    }
    *total = tot;
    return before + incl - x;
}

template <int NW>
__device__ void fused_select(const ScoreArgs &a, int row, int part, int P, int n, const uint64_t *items,
                             uint32_t *hist_s, int *scratch, uint8_t *area, int area_bytes,
                             uint64_t *ties_out_g, const uint64_t *runs_row, int run_stride) {
    constexpr int NTH = NW * 32;
    constexpr int kPmax = 256;             // parts of a row in one fused launch (<= SMs)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int *cnt_sure = reinterpret_cast<int *>(area);        // [kPmax]
    int *cnt_tie = cnt_sure + kPmax;                     // [kPmax]
    int *tie_off = cnt_tie + kPmax;                      // [kPmax]
    int *chosen = tie_off + kPmax;                       // [kPmax]
    int *misc = chosen + kPmax;                          // [64]: ok, thr[2], counters, wsum
    int *ok = misc, *thr = misc + 2, *acc = misc + 4, *wsum = misc + 16;
    uint64_t *small = reinterpret_cast<uint64_t *>(misc + 64);   // [kSmallCap]
    uint64_t *tcache = small + kSmallCap;                // the row's ties
    const int tcap = (area_bytes - (int)((uint8_t *)tcache - area)) / 8;
    uint32_t *hist_g = a.hist + (size_t)row * kHistBins;
    uint32_t *bar = a.row_bar + row;
    uint64_t *spill = a.tie_spill + (size_t)row * a.tie_cap;
    const int kap = a.kap_out;
    EpiView sv{hist_s, scratch, thr};

    // 1. this part's histogram into the row's
    for (int i = tid; i < kHistBins; i += NTH) {
        const uint32_t v = hist_s[i];
        if (v) atomicAdd(hist_g + i, v);
    }
    if (tid < 8) acc[tid] = 0;
    block_group_barrier(bar, a.bar_base + (uint32_t)P, a.wait_ns, a.st, kWhereRescore, ok);

    // 2. the row's histogram: candidates of the row, first digit of the kappa-th
    {
        const uint4 *g4 = reinterpret_cast<const uint4 *>(hist_g);
        uint4 *s4 = reinterpret_cast<uint4 *>(hist_s);
        int mine = 0;
        for (int i = tid; i < kHistBins / 4; i += NTH) {
            const uint4 v = __ldcg(g4 + i);
            s4[i] = v;
            mine += (int)(v.x + v.y + v.z + v.w);
        }
        mine = __reduce_add_sync(0xffffffffu, mine);
        if (lane == 0) atomicAdd(&acc[0], mine);
    }
    __syncthreads();
    const int n_row = acc[0];
    const bool all = n_row <= kap;
    int b1i = 0, above1 = 0;
    if (!all) find_bin_2048<NW>(hist_s, kap, wsum, thr, &b1i, &above1);
    const uint32_t b1 = (uint32_t)b1i;
    const int need1 = kap - above1;
    // this part's candidates above b1, and its ties (published through its run)
    {
        const unsigned lt = (1u << lane) - 1u;
        int sure = 0, nt = 0;
        unsigned tm_all[kRunCap / NTH];
#pragma unroll
        for (int i = 0; i < kRunCap / NTH; ++i) {
            const int e = i * NTH + tid;
            bool tie = false;
            if (e < n) {
                const uint32_t d = (uint32_t)(items[e] >> 32) >> (32 - kHistBits);
                sure += (all || d > b1) ? 1 : 0;
                tie = !all && d == b1;
            }
            tm_all[i] = __ballot_sync(0xffffffffu, tie);
            nt += __popc(tm_all[i]);
        }
        sure = __reduce_add_sync(0xffffffffu, sure);
        int base = 0;
        if (lane == 0) {
            atomicAdd(&acc[1], sure);
            if (nt) base = atomicAdd(&acc[2], nt);
        }
        base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int i = 0; i < kRunCap / NTH; ++i) {
            if ((tm_all[i] >> lane) & 1u) ties_out_g[base + __popc(tm_all[i] & lt)] = items[i * NTH + tid];
            base += __popc(tm_all[i]);
        }
    }
    __syncthreads();
    if (tid == 0) {
        a.part_cnt[((size_t)row * P + part) * 2 + 0] = acc[1];
        a.part_cnt[((size_t)row * P + part) * 2 + 1] = acc[2];
    }
    block_group_barrier(bar, a.bar_base + 2u * (uint32_t)P, a.wait_ns, a.st, kWhereRescore, ok);
    // Every block of the grid has passed its arrivals: the next kernel may set up.
    pdl_launch_dependents();
    // every block of the row has read the row's histogram: left zeroed for the next use
    if (part == 0)
        for (int i = tid; i < kHistBins / 4; i += NTH)
            reinterpret_cast<uint4 *>(hist_g)[i] = make_uint4(0u, 0u, 0u, 0u);

    // 3. every part's counts and the head of its ties, fetched together (the
    //    run areas and the counts are in L2); the ties are used in place,
    //    part p's i-th at stage[p * spec + i].  A head of 128 (64 when that
    //    does not fit) holds a part's ties nearly always: a part of ~1000
    //    candidates has ~50 of the threshold's first digit, and a part over
    //    the head costs a second round trip for the whole row.
    const int spec_sh = (long long)P * 128 <= tcap ? 7 : 6;
    const int spec = 1 << spec_sh;
    uint64_t *stage_t = tcache;                          // [P][spec]
    const bool spec_fits = (long long)P * spec <= tcap;
    if (spec_fits) {
        for (int q = tid; q < P * (spec / 2); q += NTH) {
            const int p = q >> (spec_sh - 1), e2 = 2 * (q - p * (spec / 2));
            cp_async16(stage_t + p * spec + e2, runs_row + (size_t)p * run_stride + e2, 16u);
        }
        cp_async_commit();
    }
    int cs = 0, ct = 0;
    if (tid < P) {
        cs = __ldcg(a.part_cnt + ((size_t)row * P + tid) * 2 + 0);
        ct = __ldcg(a.part_cnt + ((size_t)row * P + tid) * 2 + 1);
        cnt_sure[tid] = cs;
        cnt_tie[tid] = ct;
    }
    for (int i = tid; i < kHistBins; i += NTH) hist_s[i] = 0;   // next 11 bits of the ties
    if (tid == 0) acc[3] = 0;
    if (spec_fits) cp_async_wait<0>();
    int m;
    const int toff = block_excl_scan_fast<NW>(ct, wsum, &m);     // barrier: counts, ties in place
    if (tid < P) tie_off[tid] = toff;
    const int big = __syncthreads_or(tid < P && ct > spec);
    // The ties in one list: in place (every part's ties fit the fetched head)
    // or compacted in order into tcache / the spill (a part with more).
    const bool in_place = spec_fits && !big;
    const int nslot = in_place ? P * spec : m;
    auto tie_slot = [&](int f, uint64_t *it) -> bool {  // f-th slot of the list: a tie?
        if (in_place) {
            const int p = f >> spec_sh;
            if (f - (p << spec_sh) >= cnt_tie[p]) return false;
            *it = stage_t[f];
            return true;
        }
        *it = f < tcap ? tcache[f] : __ldcg(spill + f);
        return true;
    };
    uint32_t T = 0u;
    int cutoff = 0x7fffffff;
    if (!all && m > 0) {
        if (!in_place) {
            // compaction (into tcache, which overwrites the fetched heads)
            __syncthreads();
            for (int p = warp; p < P; p += NW) {
                const int c = cnt_tie[p], o = tie_off[p];
                for (int i = lane; i < c; i += 32) {
                    const uint64_t it = __ldcg(runs_row + (size_t)p * run_stride + i);
                    const int e = o + i;
                    if (e < tcap) tcache[e] = it;
                    else if (e < a.tie_cap) spill[e] = it;
                }
            }
            __syncthreads();
        }
        for (int f = tid; f < nslot; f += NTH) {
            uint64_t it;
            if (tie_slot(f, &it)) atomicAdd(&hist_s[((uint32_t)(it >> 32) >> 10) & 0x7ffu], 1u);
        }
        __syncthreads();
        if (need1 < m) {
            int b2, above2;
            find_bin_2048<NW>(hist_s, need1, wsum, thr, &b2, &above2);
            const int need2 = need1 - above2;
            const uint32_t hi21 = (b1 << 21) | ((uint32_t)b2 << 10);
            if ((int)hist_s[b2] <= kSmallCap) {
                for (int f = tid; f < nslot; f += NTH) {
                    uint64_t it;
                    if (tie_slot(f, &it) && ((uint32_t)(it >> 32) & 0xfffffc00u) == hi21)
                        small[atomicAdd(&acc[3], 1)] = it;
                }
                __syncthreads();
                // the need2-th item of the bin in (key descending, position ascending) order
                const int ns = acc[3];
                for (int i = tid; i < ns; i += NTH) {
                    const uint64_t u = small[i];
                    const uint32_t ku = (uint32_t)(u >> 32), pu = (uint32_t)u;
                    int rk = 0;
                    for (int j = 0; j < ns; ++j) {
                        const uint64_t w = small[j];
                        const uint32_t kw = (uint32_t)(w >> 32);
                        rk += kw > ku || (kw == ku && (uint32_t)w < pu);
                    }
                    if (rk == need2 - 1) {
                        thr[0] = (int)ku;
                        thr[1] = (int)pu;
                    }
                }
                __syncthreads();
                T = (uint32_t)thr[0];
                cutoff = thr[1];
            } else {
                if (in_place) {
                    // the histogram fallback takes the ties as one list
                    __syncthreads();
                    for (int p = warp; p < P; p += NW) {
                        const int c = cnt_tie[p], o = tie_off[p];
                        for (int i = lane; i < c; i += 32) spill[o + i] = stage_t[p * spec + i];
                    }
                    __threadfence_block();
                    __syncthreads();
                }
                auto tie_at = [&](int e) -> uint64_t {
                    return in_place ? __ldcg(spill + e) : (e < tcap ? tcache[e] : __ldcg(spill + e));
                };
                resolve_threshold(sv, tie_at, m, b1, need1, &T, &cutoff);
            }
        }
    }
    // every part's chosen ties (all of them when need1 >= m)
    for (int p = tid; p < P; p += NTH) chosen[p] = 0;
    __syncthreads();
    if (!all && m > 0) {
        if (in_place) {
            for (int f = tid; f < nslot; f += NTH) {
                uint64_t it;
                if (!tie_slot(f, &it)) continue;
                const uint32_t ku = (uint32_t)(it >> 32);
                if (ku > T || (ku == T && (int)(uint32_t)it <= cutoff)) atomicAdd(&chosen[f >> spec_sh], 1);
            }
        } else {
            for (int p = warp; p < P; p += NW) {
                const int c = cnt_tie[p], o = tie_off[p];
                int k = 0;
                for (int i = lane; i < c; i += 32) {
                    const int e = o + i;
                    const uint64_t it = e < tcap ? tcache[e] : __ldcg(spill + e);
                    const uint32_t ku = (uint32_t)(it >> 32);
                    k += (ku > T || (ku == T && (int)(uint32_t)it <= cutoff)) ? 1 : 0;
                }
                k = __reduce_add_sync(0xffffffffu, k);
                if (lane == 0) chosen[p] = k;
            }
        }
    }
    __syncthreads();
    // this part's offset in the selection, and the selection's size
    int total_sel;
    const int poff = block_excl_scan_fast<NW>(tid < P ? cnt_sure[tid] + chosen[tid] : 0, wsum, &total_sel);
    if (tid == part) acc[5] = poff;
    __syncthreads();
    const int my_off = acc[5];

    // 4. this part's selected positions, in order, at its offset: item
    //    i * NTH + t is thread t's i-th (conflict-free reads); its output
    //    index comes from the per-(round, warp) counts after one barrier
    int32_t *out = a.sel_out + (size_t)row * kap;
    auto picked = [&](uint64_t it) {
        const uint32_t ku = (uint32_t)(it >> 32);
        const uint32_t d = ku >> (32 - kHistBits);
        return all || d > b1 || (d == b1 && (ku > T || (ku == T && (int)(uint32_t)it <= cutoff)));
    };
    constexpr int R = kRunCap / NTH;
    int *rw = cnt_tie;                                   // [R][NW] counts (cnt_tie is done)
    unsigned pm[R];
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int e = i * NTH + tid;
        pm[i] = __ballot_sync(0xffffffffu, e < n && picked(items[e]));
        if (lane == 0) rw[i * NW + warp] = __popc(pm[i]);
    }
    __syncthreads();
    int o = my_off;
#pragma unroll
    for (int i = 0; i < R; ++i) {
        int before = 0, rt = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const int v = rw[i * NW + w];
            before += w < warp ? v : 0;
            rt += v;
        }
        if ((pm[i] >> lane) & 1u) {
            const int j = o + before + __popc(pm[i] & lt);
            if (j < kap) out[j] = (int)(uint32_t)items[i * NTH + tid];
        }
        o += rt;
    }
    if (part == P - 1)
        for (int j = total_sel + tid; j < kap; j += NTH) out[j] = -1;
    if (part == 0 && tid == 0 && total_sel != min(kap, n_row))
        report(a.st, kDevErrInternal, kWhereRescore, (uint32_t)total_sel);
}

template <int D, int FMT, int NT = 1, int ST = 3>
__global__ void __launch_bounds__(RescoreCfg<D, FMT, ST>::kThreads, 1)
k_refine_rescore(ScoreArgs a) {
    using C = RescoreCfg<D, FMT, ST>;
    constexpr bool MAXAGG = FMT != kFmtSum;
    constexpr int EPT = kMaxPartEntries / C::kThreads;     // source entries a thread
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *items = reinterpret_cast<uint64_t *>(smem + C::kItemOff);
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(smem + C::kHistOff);
    int *scratch = reinterpret_cast<int *>(smem + C::kScratchOff);
    const int row = blockIdx.y, part = blockIdx.x, P = gridDim.x, z = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereRescore);
    for (int i = tid; i < kHistBins; i += C::kThreads) hist_s[i] = 0;

    // This lane's query data (an input: read while the predecessor finishes).
    // Group sum: qbar, this lane's 8 elements.  Group maximum: the B fragments
    // of the group's queries (column n of n-tile t is head (8t + n) % G; k
    // pairs 2*(lane%4) and +8 of each 16-wide k step).
    const int slice = lane % C::kNL, sub = lane / C::kNL;
    const uint16_t *qb = static_cast<const uint16_t *>(z == 0 ? a.q : a.qz[z]);
    const int Hq = a.Hkv * a.G;
    float qreg[8];
    uint32_t qf[2][D / 16][2];
    Q2Query<D, NT> Q;
    if constexpr (FMT == kFmtQ2) {
        q2_load_query<D, NT>(Q, qb + ((size_t)b * Hq + (size_t)h * a.G) * D, a.G, lane);
    } else if constexpr (!MAXAGG) {
#pragma unroll
        for (int e = 0; e < 8; ++e) qreg[e] = 0.f;
        for (int g = 0; g < a.G; ++g) {
            const uint4 w = *reinterpret_cast<const uint4 *>(
                qb + ((size_t)b * Hq + (size_t)h * a.G + g) * D + slice * 8);
            qreg[0] += bf16_lo(w.x); qreg[1] += bf16_hi(w.x);
            qreg[2] += bf16_lo(w.y); qreg[3] += bf16_hi(w.y);
            qreg[4] += bf16_lo(w.z); qreg[5] += bf16_hi(w.z);
            qreg[6] += bf16_lo(w.w); qreg[7] += bf16_hi(w.w);
        }
    } else {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int head = (8 * t + (lane >> 2)) % a.G;
            const uint16_t *qh = qb + ((size_t)b * Hq + (size_t)h * a.G + head) * D + 2 * (lane & 3);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                qf[t][kk][0] = *reinterpret_cast<const uint32_t *>(qh + 16 * kk);
                qf[t][kk][1] = *reinterpret_cast<const uint32_t *>(qh + 16 * kk + 8);
            }
        }
    }
    const bool two_tiles = a.G > 8;
    __syncthreads();                                    // histogram zeroed

    // The source selection comes from the preceding kernels.
    pdl_wait();
    const int E = a.kappa;
    // the windows' global bounds and the shard they are cut to (the whole row
    // on one GPU)
    const int Lg = a.glen ? load_len(a.glen, b, a.glmax, a.st, kWhereRescore) : L;
    const long long slo = a.glen ? a.shard_lo : 0, shi = slo + L - 1;
    const int j0 = (int)((long long)part * E / P), j1 = (int)((long long)(part + 1) * E / P);
    const int ne = min(j1 - j0, kMaxPartEntries);
    const int32_t *src = a.src + (size_t)row * E + j0;
    // The ranges owned by this thread's entries [t0, t0 + EPT) of the part:
    // first slot, length, first position (kept in registers).
    const int t0 = tid * EPT;
    int cnt[EPT], lo_[EPT], off_[EPT];
    {
        int prev = (t0 < ne && j0 + t0 > 0) ? __ldcg(src + t0 - 1) : -1;
        int cur[EPT];
#pragma unroll
        for (int e = 0; e < EPT; ++e) cur[e] = t0 + e < ne ? __ldcg(src + t0 + e) : -1;
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int i = cur[e];
            cnt[e] = 0;
            lo_[e] = 0;
            if (i >= 0) {
                if (i >= Lg || (prev >= 0 && i <= prev)) {
                    report(a.st, kDevErrBadIndex, kWhereRescore, (uint32_t)i);
                } else {
                    long long lo = (long long)i - a.radius;
                    if (prev >= 0 && (long long)prev + a.radius + 1 > lo) lo = (long long)prev + a.radius + 1;
                    if (lo < 0) lo = 0;
                    long long hi = (long long)i + a.radius;
                    if (hi > Lg - 1) hi = Lg - 1;
                    if (lo < slo) lo = slo;
                    if (hi > shi) hi = shi;
                    if (hi >= lo) {
                        lo_[e] = (int)(lo - slo);
                        cnt[e] = (int)(hi - lo + 1);
                    }
                }
            }
            prev = i;
        }
    }
    int n;
    {
        int mine = 0;
#pragma unroll
        for (int e = 0; e < EPT; ++e) mine += cnt[e];
        int run = block_exclusive_scan(mine, scratch, &n);
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            off_[e] = run;
            run += cnt[e];
        }
    }
    const int K = a.run_k;
    if (n > K * kRunCap) {
        if (tid == 0) report(a.st, kDevErrInternal, kWhereRescore, (uint32_t)n);
        n = K * kRunCap;
    }

    const uint8_t *kb = static_cast<const uint8_t *>(z == 0 ? a.k : a.kz[z]) +
                        (size_t)row * a.Lmax * C::kRowBytes;
    const size_t nruns = (size_t)P * K;
    uint64_t *runs_row = a.runs + (size_t)z * a.zruns + (size_t)row * nruns * kRunCap;
    int32_t *cnt_row = a.run_cnt + (size_t)z * a.zcnt + (size_t)row * nruns;
    uint32_t *hist_g = a.hist + (size_t)z * a.zhist + (size_t)row * kHistBins;
    float *Spos = a.Spos ? a.Spos + (size_t)row * a.spos_stride : nullptr;
    const int r_base = warp * C::kRowsPerWarp;
    // The row (of the warp's 16) whose score this lane stores, if it is a writer.
    const int rr_item = MAXAGG ? (lane >> 2) + ((lane & 3) == 1 ? 8 : 0)
                               : transpose_item<C::kSteps, C::kNL>(lane) * C::kRPI + sub;
    const bool writer = MAXAGG ? (lane & 3) < 2 : transpose_writer<C::kSteps, C::kNL>(lane);
    uint32_t *item_w = reinterpret_cast<uint32_t *>(items);   // [2e]: position, [2e + 1]: key
    const int last = n > 0 ? (n - 1) / kRunCap : -1;

    for (int k = 0; k <= last; ++k) {
        const int s0 = k * kRunCap;
        const int nk = min(kRunCap, n - s0);
        // The run's position table.
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int a0 = max(off_[e], s0), a1 = min(off_[e] + cnt[e], s0 + nk);
            for (int t = a0; t < a1; ++t) item_w[2 * (t - s0)] = (uint32_t)(lo_[e] + (t - off_[e]));
        }
        __syncthreads();
        const int nwin = (nk + C::kTileRows - 1) / C::kTileRows;
        // This lane's pieces of window w (rows st*kRPI + sub of the warp's 16,
        // bytes [16*slice, 16*slice + 16)); rows past the run are zero-filled.
        auto gather = [&](int w) {
            const int first = w * C::kTileRows + r_base;
            uint8_t *dst = stages + ((w % C::kStages) * C::kWarps + warp) * C::kWarpStage + slice * 16;
#pragma unroll
            for (int sp = 0; sp < C::kSteps; ++sp) {
                const int rr = sp * C::kRPI + sub;
                const bool ok = first + rr < nk;
                const int p = ok ? (int)item_w[2 * (first + rr)] : 0;
                cp_async16(dst + rr * C::kRowStride, kb + (size_t)p * C::kRowBytes + slice * 16, ok ? 16u : 0u);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int w = 0; w < C::kStages - 1; ++w) {
            if (w < nwin) gather(w);
            else cp_async_commit();
        }
        for (int w = 0; w < nwin; ++w) {
            if (w + C::kStages - 1 < nwin) gather(w + C::kStages - 1);
            else cp_async_commit();
            cp_async_wait<C::kStages - 1>();             // this lane's pieces of window w
            const uint8_t *tw = stages + ((w % C::kStages) * C::kWarps + warp) * C::kWarpStage;
            float part_[C::kSteps];
            if constexpr (FMT == kFmtQ2) {
                __syncwarp();                            // the warp reads rows of all its lanes
                const float2 m = q2_group_max_16rows<D, NT>(tw, Q, lane);
                part_[0] = (lane & 3) == 1 ? m.y : m.x;
            } else if constexpr (MAXAGG) {
                __syncwarp();
                const float2 m = group_max_16rows<D, C::kRowStride>(tw, qf, two_tiles, lane);
                part_[0] = (lane & 3) == 1 ? m.y : m.x;
            } else {
#pragma unroll
                for (int sp = 0; sp < C::kSteps; ++sp) {
                    const uint4 kv = *reinterpret_cast<const uint4 *>(
                        tw + (sp * C::kRPI + sub) * C::kRowStride + slice * 16);
                    part_[sp] = dot8(kv, qreg);
                }
                transpose_reduce<C::kSteps, C::kNL>(part_, lane);
            }
            __syncwarp();                                // the stage is free for the next gather
            const int t = w * C::kTileRows + r_base + rr_item;     // run-local slot
            if (writer && t < nk) {
                const float sc = part_[0] * a.scale;
                const uint32_t key = score_key(sc);
                item_w[2 * t + 1] = key;
                atomicAdd(&hist_s[key >> (32 - kHistBits)], 1u);
                if (Spos) Spos[item_w[2 * t]] = sc;
            }
        }
        cp_async_wait<0>();
        __syncthreads();                         // every copy landed, every key in place
        if (a.fused) break;                      // one run: the fused selection below
        // The selection may set up now; it waits for this grid before reading.
        if (k == last) pdl_launch_dependents();

        // Counting sort of the run by first digit, highest first: this run's
        // histogram goes to the row's and becomes the bins' start offsets.
        constexpr int BPT = kHistBins / C::kThreads;
        const int hb = kHistBins - (tid + 1) * BPT;   // thread 0 owns the top bins
        uint32_t hv[BPT];
        int mine = 0;
#pragma unroll
        for (int i = 0; i < BPT; ++i) {
            hv[i] = hist_s[hb + i];
            mine += (int)hv[i];
            if (hv[i]) atomicAdd(hist_g + hb + i, hv[i]);
        }
        int tot;
        int cur = block_exclusive_scan(mine, scratch, &tot);   // items in higher bins
#pragma unroll
        for (int i = BPT - 1; i >= 0; --i) {
            hist_s[hb + i] = (uint32_t)cur;
            cur += (int)hv[i];
        }
        __syncthreads();
        uint64_t *dst_g = runs_row + (size_t)(part * K + k) * kRunCap;
        uint64_t *dst = C::kStageSort ? reinterpret_cast<uint64_t *>(stages) : dst_g;
        for (int e = tid; e < nk; e += C::kThreads) {
            const uint64_t it = items[e];
            const uint32_t o = atomicAdd(&hist_s[(uint32_t)(it >> 32) >> (32 - kHistBits)], 1u);
            if (o < (uint32_t)nk) dst[o] = it;
        }
        __syncthreads();
        if constexpr (C::kStageSort) {
            const uint4 *s4 = reinterpret_cast<const uint4 *>(stages);
            uint4 *d4 = reinterpret_cast<uint4 *>(dst_g);
            for (int e = tid; 2 * e < nk; e += C::kThreads) {
                if (2 * e + 1 < nk) d4[e] = s4[e];
                else dst_g[2 * e] = reinterpret_cast<const uint64_t *>(stages)[2 * e];
            }
        }
        if (tid == 0) cnt_row[part * K + k] = nk;
        for (int i = tid; i < kHistBins; i += C::kThreads) hist_s[i] = 0;
        __syncthreads();                         // stages, table and histogram free again
    }
    if (a.fused) {
        fused_select<C::kWarps>(a, row, part, P, n, items, hist_s, scratch, stages, C::kStageBytes,
                                runs_row + (size_t)part * K * kRunCap, runs_row, K * kRunCap);
        return;
    }
    if (last < 0) pdl_launch_dependents();
    if (tid == 0)
        for (int k = last + 1; k < K; ++k) cnt_row[part * K + k] = 0;
}

// ---------------------------------------------------------------------------
template <int D>
static cudaError_t launch_anchor_score_d(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    using C = AnchorCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(k_anchor_score<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.Hkv;
    const long long max_tiles = rows * ((a.Lmax + C::kTileRows - 1) / C::kTileRows);
    const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
    return launch_kernel(k_anchor_score<D>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, s, a);
}

cudaError_t launch_anchor_score(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    if (a.agg == kAggMax && a.q2) return launch_anchor_score_q2(a, num_sms, s);
    if (a.agg == kAggMax) return launch_anchor_score_max(a, num_sms, s);
    return a.d == 128 ? launch_anchor_score_d<128>(a, num_sms, s)
                      : launch_anchor_score_d<64>(a, num_sms, s);
}


template <int D, int FMT, int NT = 1, int ST = 3>
static cudaError_t launch_refine_rescore_d(const ScoreArgs &a, cudaStream_t s) {
    using C = RescoreCfg<D, FMT, ST>;
    cudaError_t e = cudaFuncSetAttribute(k_refine_rescore<D, FMT, NT, ST>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int nz = a.nz > 1 ? a.nz : 1;
    const int rows = a.B * a.Hkv;
    return launch_kernel(k_refine_rescore<D, FMT, NT, ST>, dim3((unsigned)a.parts, (unsigned)rows, (unsigned)nz),
                         dim3(C::kThreads), C::kSmemBytes, s, a);
}

cudaError_t launch_refine_rescore(const ScoreArgs &a, cudaStream_t s) {
    if (a.parts < 1 || a.run_k < 1 || (long long)(a.kappa + a.parts - 1) / a.parts > kMaxPartEntries)
        return cudaErrorInvalidValue;
    if (a.agg == kAggMax && a.q2) {
        if (a.G > 8)
            return a.d == 128 ? launch_refine_rescore_d<128, kFmtQ2, 2>(a, s)
                              : launch_refine_rescore_d<64, kFmtQ2, 2>(a, s);
        return a.d == 128 ? launch_refine_rescore_d<128, kFmtQ2, 1>(a, s)
                          : launch_refine_rescore_d<64, kFmtQ2, 1>(a, s);
    }
    if (a.agg == kAggMax)
        return a.d == 128 ? launch_refine_rescore_d<128, kFmtMax>(a, s)
                          : launch_refine_rescore_d<64, kFmtMax>(a, s);
    if (a.two_stages)
        return a.d == 128 ? launch_refine_rescore_d<128, kFmtSum, 1, 2>(a, s)
                          : launch_refine_rescore_d<64, kFmtSum, 1, 2>(a, s);
    return a.d == 128 ? launch_refine_rescore_d<128, kFmtSum>(a, s)
                      : launch_refine_rescore_d<64, kFmtSum>(a, s);
}

}  // namespace prism
