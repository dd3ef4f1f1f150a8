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
// Refined layer: score only the proposal positions (Eq. (5)).  The proposal
// of a row is enumerated slot by slot from the owned ranges of the canonical
// source selection (the offsets src_off give each entry's first slot), so a
// row's n slots split evenly into P contiguous parts, one CTA each.  A CTA
// walks its part in windows of 128 slots.  The producer warp finds the
// entries overlapping each window (one coalesced load of 32 entries at a
// time, the next batch in flight) and writes every slot's key row into a ring
// of position tables, up to kPosDepth windows ahead.  Each consumer warp owns
// 16 slots of every window: it gathers exactly the 16-byte pieces of those
// key rows that its lanes will read (cp.async, a 3-stage pipeline per warp,
// no hand-off between warps), forms the dot products and stores the
// (score, position) candidates at their slot index.  (A run of the proposal
// is only ~11-17 rows, 3-4 KB: issuing one bulk copy per run from a single
// warp, not DRAM, limited an earlier version to ~25 GB/s per SM.)
// Key formats of the rescoring kernel: bf16 keys with the group sum
// (Eq. (1)), bf16 keys with the group maximum (Eq. (9)), 2-bit keys with the
// group maximum (Eq. (7)-(9), row format of q2_impl.cuh).
enum : int { kFmtSum = 0, kFmtMax = 1, kFmtQ2 = 2 };

template <int D, int FMT = kFmtSum>
struct RescoreCfg {
    static constexpr int kTileRows = 128;
    static constexpr int kStages = 3;                  // data stages per consumer warp
    static constexpr int kPosDepth = 8;                // position tables in the ring
    static constexpr int kConsumerWarps = 8;
    static constexpr int kThreads = 32 * (kConsumerWarps + 1);
    static constexpr int kRowBytes = FMT == kFmtQ2 ? q2_row_bytes(D) : D * 2;
    static constexpr int kNL = kRowBytes / 16;         // lanes (16-byte pieces) per key row
    static constexpr int kRPI = 32 / kNL;
    static constexpr int kRowsPerWarp = kTileRows / kConsumerWarps;   // 16
    static constexpr int kSteps = kRowsPerWarp / kRPI;
    static constexpr int kTileBytes = kTileRows * kRowBytes;
    static constexpr int kPosOff = kStages * kTileBytes;
    static constexpr int kBarOff = kPosOff + kPosDepth * kTileRows * 4;
    static constexpr int kHistOff = kBarOff + 2 * kPosDepth * 8;
    static constexpr int kSmemBytes = kHistOff + kHistBins * 4;
};

// Group maximum (Eq. (9) form) of a warp's 16 gathered rows: the [16 x d] x
// [d x 8] products of mma.sync m16n8k16 (bf16 in, fp32 accumulate; one or two
// n-tiles of 8 heads), A fragments by ldmatrix from rows whose 16-byte chunk c
// sits at chunk c ^ (row % 8) (conflict-free), B fragments (the group's
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
template <int D>
__device__ __forceinline__ float2 group_max_16rows(const uint8_t *rows16, const uint32_t (&qf)[2][D / 16][2],
                                                   bool two_tiles, int lane) {
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
    const int r = (lane & 7) + ((lane >> 3) & 1) * 8;       // row this lane addresses
    const uint32_t base = smem_addr(rows16 + r * (D * 2));
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int chunk = 2 * kk + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(base + (uint32_t)((chunk ^ (lane & 7)) << 4), a0, a1, a2, a3);
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

template <int D, int FMT, int NT = 1>
__global__ void __launch_bounds__(RescoreCfg<D, FMT>::kThreads, 1)
k_refine_rescore(ScoreArgs a) {
    using C = RescoreCfg<D, FMT>;
    constexpr bool MAXAGG = FMT != kFmtSum;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    int *pos_s = reinterpret_cast<int *>(smem + C::kPosOff);
    uint64_t *pos_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *pos_empty = pos_full + C::kPosDepth;
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(smem + C::kHistOff);
    const int row = blockIdx.y, part = blockIdx.x, P = gridDim.x, z = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int cstride = a.cstride > 0 ? a.cstride : a.Lmax;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereRescore);
    for (int i = tid; i < kHistBins; i += C::kThreads) hist_s[i] = 0;
    if (tid == 0) {
        for (int s = 0; s < C::kPosDepth; ++s) {
            mbar_init(&pos_full[s], 1);
            mbar_init(&pos_empty[s], C::kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    // The source selection and its offsets come from the preceding kernels.
    pdl_wait();
    const int32_t *off = a.src_off + (size_t)row * (a.kappa + 1);
    const int n = min(min(__ldcg(off + a.kappa), L), a.Lmax);
    const int s_begin = (int)((long long)part * n / P);
    const int s_end = (int)((long long)(part + 1) * n / P);
    const int nwin = (s_end - s_begin + C::kTileRows - 1) / C::kTileRows;
    if (nwin <= 0) {
        pdl_launch_dependents();
        return;
    }

    if (warp == C::kConsumerWarps) {
        // ---------------- producer warp: the position tables ---------------------
        const int32_t *src = a.src + (size_t)row * a.kappa;
        if (a.radius == 0) {
            // Radius 0 (a pool, or a proposal already cut into single
            // positions): each entry of the canonical source owns exactly its
            // own position, so slot s is entry s and a window's table is a
            // copy of the source.  A malformed entry (outside [0, L), or not
            // above its predecessor) is reported and reads row 0.
            for (int it = 0; it < nwin; ++it) {
                const int s = it % C::kPosDepth;
                const uint32_t ph = (uint32_t)(it / C::kPosDepth) & 1u;
                if (!mbar_wait(&pos_empty[s], ph ^ 1u, a.wait_ns)) {
                    if (lane == 0) report(a.st, kDevErrTimeout, kWhereRescore, (uint32_t)it);
                    break;
                }
                const int w0 = s_begin + it * C::kTileRows;
                const int wend = min(w0 + C::kTileRows, s_end);
                int *pos = pos_s + s * C::kTileRows;
                for (int t = w0 + lane; t < wend; t += 32) {
                    int p = __ldcg(src + t);
                    const int prev = t > 0 ? __ldcg(src + t - 1) : -1;
                    if (p < 0 || p >= L || p <= prev) {
                        report(a.st, kDevErrBadIndex, kWhereRescore, (uint32_t)p);
                        p = 0;
                    }
                    pos[t - w0] = p;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&pos_full[s]);
            }
            return;
        }
        // First entry to look at: the last one starting at or before s_begin,
        // by a 64-way search over the offsets (off[0] = 0 <= s_begin).
        int lo = 0, hi = a.kappa;
        while (hi - lo > 32) {
            const int st = (hi - lo + 63) / 64;
            const int x0 = lo + 2 * lane * st, x1 = x0 + st;
            const bool p0 = x0 < hi && __ldcg(off + x0) <= s_begin;
            const bool p1 = x1 < hi && __ldcg(off + x1) <= s_begin;
            const unsigned m0 = __ballot_sync(0xffffffffu, p0), m1 = __ballot_sync(0xffffffffu, p1);
            const int k0 = m0 ? 2 * (31 - __clz(m0)) : 0;
            const int k1 = m1 ? 2 * (31 - __clz(m1)) + 1 : 0;
            lo += max(k0, k1) * st;
            hi = min(hi, lo + st);
        }
        int jb = lo;
        EntryRun e = make_entry(load_entry_raw(src, off, a.kappa, jb + lane), jb + lane, a.kappa, n,
                                a.radius, L, a.st);
        EntryRaw next = load_entry_raw(src, off, a.kappa, jb + 32 + lane);
        for (int it = 0; it < nwin; ++it) {
            const int s = it % C::kPosDepth;
            const uint32_t ph = (uint32_t)(it / C::kPosDepth) & 1u;
            if (!mbar_wait(&pos_empty[s], ph ^ 1u, a.wait_ns)) {
                if (lane == 0) report(a.st, kDevErrTimeout, kWhereRescore, (uint32_t)it);
                break;
            }
            const int w0 = s_begin + it * C::kTileRows;
            const int wend = min(w0 + C::kTileRows, s_end);
            int *pos = pos_s + s * C::kTileRows;
            for (;;) {
                const int g0 = max(e.o0, w0), g1 = min(e.o1, wend);
                if (g0 < g1) {
                    // keep the rows inside this row of the key cache whatever the offsets say
                    const int r0 = min(e.lo + (g0 - e.o0), a.Lmax - (g1 - g0));
                    for (int t = g0; t < g1; ++t) pos[t - w0] = r0 + (t - g0);
                }
                const int reach = __shfl_sync(0xffffffffu, e.o1, 31);
                if (reach >= wend || jb + 32 >= a.kappa) break;
                jb += 32;
                e = make_entry(next, jb + lane, a.kappa, n, a.radius, L, a.st);
                next = load_entry_raw(src, off, a.kappa, jb + 32 + lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pos_full[s]);
        }
        return;
    }

    // ---------------- consumers ------------------------------------------------
    const int slice = lane % C::kNL, sub = lane / C::kNL;
    const uint16_t *qb = static_cast<const uint16_t *>(z == 0 ? a.q : a.qz[z]);
    const int Hq = a.Hkv * a.G;
    // Group sum: qbar, this lane's 8 elements.  Group maximum: the B fragments
    // of the group's queries (column n of n-tile t is head (8t + n) % G; k
    // pairs 2*(lane%4) and +8 of each 16-wide k step).
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
    const uint8_t *kb = static_cast<const uint8_t *>(z == 0 ? a.k : a.kz[z]) +
                        (size_t)row * a.Lmax * C::kRowBytes;
    float *S = a.S + (size_t)z * a.zS + (size_t)row * cstride;
    int32_t *cpos = a.cpos + (size_t)z * a.zS + (size_t)row * cstride;
    const int r_base = warp * C::kRowsPerWarp;
    // The row whose score this lane stores, if it is a writer.
    const int r_item = MAXAGG ? r_base + (lane >> 2) + ((lane & 3) == 1 ? 8 : 0)
                              : r_base + transpose_item<C::kSteps, C::kNL>(lane) * C::kRPI + sub;
    const bool writer = MAXAGG ? (lane & 3) < 2 : transpose_writer<C::kSteps, C::kNL>(lane);
    bool failed = false;
    // Issue this lane's pieces of window `it` (rows r_base + st*kRPI + sub,
    // bytes [16*slice, 16*slice + 16)); rows past the window are zero-filled.
    auto gather = [&](int it) {
        const int s = it % C::kPosDepth;
        const uint32_t ph = (uint32_t)(it / C::kPosDepth) & 1u;
        if (!failed && !mbar_wait(&pos_full[s], ph, a.wait_ns)) {
            if (lane == 0) report(a.st, kDevErrTimeout, kWhereRescore, 0x40000000u | (uint32_t)it);
            failed = true;
        }
        const int nrows = min(C::kTileRows, s_end - (s_begin + it * C::kTileRows));
        const int *pos = pos_s + s * C::kTileRows;
        uint8_t *tile = stages + (it % C::kStages) * C::kTileBytes;
#pragma unroll
        for (int st = 0; st < C::kSteps; ++st) {
            const int r = r_base + st * C::kRPI + sub;
            const bool ok = !failed && r < nrows;
            const int krow = ok ? pos[r] : 0;
            // the bf16 group-maximum path reads the rows by ldmatrix: swizzled chunks
            const int chunk = FMT == kFmtMax ? (slice ^ (r & 7)) : slice;
            cp_async16(tile + r * C::kRowBytes + chunk * 16,
                       kb + (size_t)krow * C::kRowBytes + slice * 16, ok ? 16u : 0u);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int it = 0; it < C::kStages - 1; ++it) {
        if (it < nwin) gather(it);
        else cp_async_commit();
    }
    for (int it = 0; it < nwin; ++it) {
        if (it + C::kStages - 1 < nwin) gather(it + C::kStages - 1);
        else cp_async_commit();
        cp_async_wait<C::kStages - 1>();                // this lane's pieces of window `it`
        const uint8_t *tile = stages + (it % C::kStages) * C::kTileBytes;
        float part_[C::kSteps];
        if constexpr (FMT == kFmtQ2) {
            // The warp reads rows gathered by all of its lanes.
            __syncwarp();
            const float2 m = q2_group_max_16rows<D, NT>(tile + r_base * C::kRowBytes, Q, lane);
            part_[0] = (lane & 3) == 1 ? m.y : m.x;
        } else if constexpr (MAXAGG) {
            // The warp reads rows gathered by all of its lanes.
            __syncwarp();
            const float2 m = group_max_16rows<D>(tile + r_base * C::kRowBytes, qf, two_tiles, lane);
            part_[0] = (lane & 3) == 1 ? m.y : m.x;
        } else {
#pragma unroll
            for (int st = 0; st < C::kSteps; ++st) {
                const int r = r_base + st * C::kRPI + sub;
                const uint4 kv = *reinterpret_cast<const uint4 *>(tile + r * C::kRowBytes + slice * 16);
                part_[st] = dot8(kv, qreg);
            }
        }
        const int s = it % C::kPosDepth;
        const int p_item = pos_s[s * C::kTileRows + r_item];
        __syncwarp();
        if (lane == 0) mbar_arrive(&pos_empty[s]);
        if constexpr (!MAXAGG) transpose_reduce<C::kSteps, C::kNL>(part_, lane);
        const int w0 = s_begin + it * C::kTileRows;
        const int nrows = min(C::kTileRows, s_end - w0);
        if (!failed && writer && r_item < nrows) {
            const float sc = part_[0] * a.scale;
            S[w0 + r_item] = sc;
            cpos[w0 + r_item] = p_item;
            atomicAdd(&hist_s[score_key(sc) >> (32 - kHistBits)], 1u);
        }
    }
    cp_async_wait<0>();
    consumer_sync();
    pdl_launch_dependents();
    uint32_t *hist_g = a.hist + (size_t)z * a.zhist + (size_t)row * kHistBins;
    for (int i = tid; i < kHistBins; i += 32 * C::kConsumerWarps) {
        const uint32_t v = hist_s[i];
        if (v) atomicAdd(hist_g + i, v);
    }
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


template <int D, int FMT, int NT = 1>
static cudaError_t launch_refine_rescore_d(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    using C = RescoreCfg<D, FMT>;
    cudaError_t e = cudaFuncSetAttribute(k_refine_rescore<D, FMT, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // About one CTA per SM over all rows (of all batched layers); each row's
    // proposal is split evenly.
    const int nz = a.nz > 1 ? a.nz : 1;
    const int rows = a.B * a.Hkv;
    const int parts = rows * nz >= num_sms ? 1 : num_sms / (rows * nz);
    return launch_kernel(k_refine_rescore<D, FMT, NT>, dim3((unsigned)parts, (unsigned)rows, (unsigned)nz),
                         dim3(C::kThreads), C::kSmemBytes, s, a);
}

cudaError_t launch_refine_rescore(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    if (a.agg == kAggMax && a.q2) {
        if (a.G > 8)
            return a.d == 128 ? launch_refine_rescore_d<128, kFmtQ2, 2>(a, num_sms, s)
                              : launch_refine_rescore_d<64, kFmtQ2, 2>(a, num_sms, s);
        return a.d == 128 ? launch_refine_rescore_d<128, kFmtQ2, 1>(a, num_sms, s)
                          : launch_refine_rescore_d<64, kFmtQ2, 1>(a, num_sms, s);
    }
    if (a.agg == kAggMax)
        return a.d == 128 ? launch_refine_rescore_d<128, kFmtMax>(a, num_sms, s)
                          : launch_refine_rescore_d<64, kFmtMax>(a, num_sms, s);
    return a.d == 128 ? launch_refine_rescore_d<128, kFmtSum>(a, num_sms, s)
                      : launch_refine_rescore_d<64, kFmtSum>(a, num_sms, s);
}

}  // namespace prism
