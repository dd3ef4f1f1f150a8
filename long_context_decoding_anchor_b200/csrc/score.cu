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
// 4-stage shared-memory ring with a 1-D bulk copy (TMA, cp.async.bulk) that
// completes on an mbarrier, and eight consumer warps form the dot products
// from shared memory.  Scores go to global memory (they stay L2-resident for
// the selection) and their top 11 key bits into a per-row histogram, the
// first radix digit of the top-kappa selection.
//
// k_refine_rescore scores only the proposal positions of a refined layer
// (Eq. (5)), enumerated from the owned ranges of the source selection; each
// owned range is one bulk copy, and scores are stored by position.
#include "prism_internal.cuh"

namespace prism {

template <int D>
struct AnchorCfg {
    static constexpr int kTileRows = 128;
    static constexpr int kStages = 4;
    static constexpr int kConsumerWarps = 8;
    static constexpr int kThreads = 32 * (kConsumerWarps + 1);
    static constexpr int kNL = D / 8;                     // lanes per key row (16 B each)
    static constexpr int kRPI = 32 / kNL;                 // key rows per warp instruction
    static constexpr int kRowsPerWarp = kTileRows / kConsumerWarps;
    static constexpr int kSteps = kRowsPerWarp / kRPI;    // partial sums per lane per tile
    static constexpr int kTileBytes = kTileRows * D * 2;
    static constexpr int kSmemBytes = kStages * kTileBytes + 2 * kStages * 8 + kHistBins * 4 + 64 * 4;
};

// Position of tile `t` of the global tile order (row-major over (b, h), then
// tile j) given tiles_b = ceil(len[b] / TILE).  Found by a block-wide scan over
// the batch; every thread of the block gets the result.
struct TileCursor {
    int b, h, j, tiles_b;
};

template <int TILE>
__device__ void locate_tile(const int32_t *len, int B, int Hkv, int Lmax, long long t,
                            TileCursor *cur, long long *total, int *scratch, DevStatus *st) {
    long long base = 0;  // tiles of all (b, h) before the current batch chunk
    __shared__ long long s_found_base;
    __shared__ int s_found_b;
    __syncthreads();   // earlier readers of s_found_b are done
    if (threadIdx.x == 0) s_found_b = -1;
    __syncthreads();
    for (int b0 = 0; b0 < B; b0 += blockDim.x) {
        const int b = b0 + threadIdx.x;
        int tb = 0;
        if (b < B) {
            int L = load_len(len, b, Lmax, st, kWhereScore);
            tb = (L + TILE - 1) / TILE;
        }
        int tot;
        int ex = block_exclusive_scan(tb, scratch, &tot);
        long long my0 = base + (long long)ex * Hkv;
        long long my1 = my0 + (long long)tb * Hkv;
        if (b < B && tb > 0 && t >= my0 && t < my1) {
            s_found_b = b;
            s_found_base = my0;
        }
        base += (long long)tot * Hkv;
    }
    __syncthreads();
    *total = base;
    if (s_found_b >= 0) {
        const int b = s_found_b;
        int L = __ldg(len + b);
        L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
        const int tb = (L + TILE - 1) / TILE;
        const long long rem = t - s_found_base;
        cur->b = b;
        cur->h = (int)(rem / tb);
        cur->j = (int)(rem % tb);
        cur->tiles_b = tb;
    } else {
        cur->b = B;
        cur->h = 0;
        cur->j = 0;
        cur->tiles_b = 0;
    }
}

// Advance to the next tile (skipping empty sequences).
template <int TILE>
__device__ __forceinline__ void next_tile(TileCursor &c, const int32_t *len, int B, int Hkv,
                                          int Lmax) {
    if (++c.j < c.tiles_b) return;
    c.j = 0;
    if (++c.h < Hkv) return;
    c.h = 0;
    for (++c.b; c.b < B; ++c.b) {
        int L = __ldg(len + c.b);
        L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
        c.tiles_b = (L + TILE - 1) / TILE;
        if (c.tiles_b > 0) return;
    }
}

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
    if (t_begin >= t_end) return;
    {
        long long tot2;
        locate_tile<TILE>(a.len, a.B, a.Hkv, a.Lmax, t_begin, &cur0, &tot2, scratch, a.st);
    }
    const int ntiles = (int)(t_end - t_begin);

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
    if (cur_row >= 0) {
        for (int i = tid; i < kHistBins; i += 32 * C::kConsumerWarps) {
            uint32_t v = hist_s[i];
            if (v) atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
        }
    }
}

// ---------------------------------------------------------------------------
// Refined layer: score only the proposal positions (Eq. (5)).  One CTA per 16
// entries of the (canonical) source selection.  Each entry owns a contiguous
// run of key rows, so the gather is one 1-D bulk copy (TMA) per run, issued by
// 16 lanes of warp 0 into a shared-memory buffer that completes on an
// mbarrier; nothing is held in registers while the copies fly.  The eight
// warps then form 32 dot products per round each from shared memory, and the
// transposing reduction leaves one score per lane, stored by position.
template <int D>
struct RescoreCfg {
    static constexpr int kEntries = 16;
    static constexpr int kWarps = 8;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kNL = D / 8;
    static constexpr int kRPI = 32 / kNL;
    static constexpr int kRowsPerWarp = 32;
    static constexpr int kSteps = kRowsPerWarp / kRPI;       // == kNL
    static constexpr int kRowBytes = D * 2;
    static constexpr int kCapRows = 48 * 1024 / kRowBytes;    // rows staged per round
    static constexpr int kSmemBytes = kCapRows * kRowBytes;
    static_assert(kSteps == kNL, "one score per lane after the reduction");
};

template <int D>
__global__ void __launch_bounds__(RescoreCfg<D>::kThreads)
k_refine_rescore(ScoreArgs a) {
    using C = RescoreCfg<D>;
    extern __shared__ __align__(128) uint8_t rows_s[];
    __shared__ uint64_t bar;
    __shared__ uint32_t hist_s[kHistBins];
    __shared__ int lo_s[C::kEntries], cnt_s[C::kEntries], off_s[C::kEntries + 1];
    __shared__ int pos_s[C::kCapRows];
    __shared__ int fail_s;
    const int row = blockIdx.y;
    const int j0 = blockIdx.x * C::kEntries;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereRescore);
    const int32_t *src = a.src + (size_t)row * a.kappa;

    if (warp == 0) {
        int lo = 0, cnt = 0;
        if (lane < C::kEntries && j0 + lane < a.kappa)
            cnt = owned_range(src, j0 + lane, a.radius, L, &lo, a.st, kWhereRescore);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane < C::kEntries) {
            lo_s[lane] = lo;
            cnt_s[lane] = cnt;
            off_s[lane] = incl - cnt;
        }
        if (lane == C::kEntries - 1) off_s[C::kEntries] = incl;
        if (lane == 0) {
            fail_s = 0;
            mbar_init(&bar, 1);
            fence_mbar_init();
        }
    }
    for (int i = tid; i < kHistBins; i += C::kThreads) hist_s[i] = 0;
    __syncthreads();
    const int total = off_s[C::kEntries];
    if (total == 0) return;
    if (tid == 0) atomicAdd(&a.ctl[row].n_prop, total);

    const int slice = lane % C::kNL, sub = lane / C::kNL;
    float qreg[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qreg[e] = 0.f;
    const uint16_t *qb = static_cast<const uint16_t *>(a.q);
    const int Hq = a.Hkv * a.G;
    for (int g = 0; g < a.G; ++g) {
        const uint4 w = *reinterpret_cast<const uint4 *>(
            qb + ((size_t)b * Hq + (size_t)h * a.G + g) * D + slice * 8);
        qreg[0] += bf16_lo(w.x); qreg[1] += bf16_hi(w.x);
        qreg[2] += bf16_lo(w.y); qreg[3] += bf16_hi(w.y);
        qreg[4] += bf16_lo(w.z); qreg[5] += bf16_hi(w.z);
        qreg[6] += bf16_lo(w.w); qreg[7] += bf16_hi(w.w);
    }
    const uint16_t *kb = static_cast<const uint16_t *>(a.k) + (size_t)row * a.Lmax * D;
    float *S = a.S + (size_t)row * a.Lmax;

    int round = 0;
    bool pending = false;      // warp 0 lane 0: a round's copies may still be in flight
    for (int e0 = 0; e0 < total; e0 += C::kCapRows, ++round) {
        const int nr = min(C::kCapRows, total - e0);
        for (int i = tid; i < nr; i += C::kThreads) {
            int t = 0;                                  // entry owning index e0 + i
#pragma unroll
            for (int m = 8; m >= 1; m >>= 1)
                if (t + m < C::kEntries && off_s[t + m] <= e0 + i) t += m;
            pos_s[i] = lo_s[t] + (e0 + i - off_s[t]);
        }
        if (warp == 0) {
            if (lane == 0) mbar_arrive_expect_tx(&bar, (uint32_t)nr * C::kRowBytes);
            __syncwarp();
            if (lane < C::kEntries) {
                const int s0 = max(off_s[lane], e0);
                const int s1 = min(off_s[lane] + cnt_s[lane], e0 + nr);
                if (s0 < s1) {
                    const uint64_t pol = l2_evict_first_policy();
                    bulk_load(rows_s + (size_t)(s0 - e0) * C::kRowBytes,
                              kb + (size_t)(lo_s[lane] + s0 - off_s[lane]) * D,
                              (uint32_t)(s1 - s0) * C::kRowBytes, &bar, pol);
                }
            }
            pending = true;
        }
        __syncthreads();                                 // pos_s ready
        const bool ok = mbar_wait(&bar, (uint32_t)round & 1u, a.wait_ns);
        if (!ok) {
            report(a.st, kDevErrTimeout, kWhereRescore, (uint32_t)round);
            fail_s = 1;
        } else {
            if (warp == 0) pending = false;
            for (int r0 = warp * C::kRowsPerWarp; r0 < nr; r0 += C::kWarps * C::kRowsPerWarp) {
                float part[C::kSteps];
#pragma unroll
                for (int st = 0; st < C::kSteps; ++st) {
                    const int r = r0 + st * C::kRPI + sub;
                    const uint4 kv = *reinterpret_cast<const uint4 *>(
                        rows_s + (size_t)r * C::kRowBytes + slice * 16);
                    part[st] = dot8(kv, qreg);
                }
                transpose_reduce<C::kSteps, C::kNL>(part, lane);
                const int r = r0 + transpose_item<C::kSteps, C::kNL>(lane) * C::kRPI + sub;
                if (r < nr) {
                    const float sc = part[0] * a.scale;
                    S[pos_s[r]] = sc;
                    atomicAdd(&hist_s[score_key(sc) >> (32 - kHistBits)], 1u);
                }
            }
        }
        __syncthreads();                                 // buffer and pos_s free again
        if (fail_s) break;
    }
    if (fail_s) {
        // Let any copy still in flight land before the CTA's shared memory goes.
        if (tid == 0 && pending && !mbar_wait(&bar, (uint32_t)round & 1u, a.wait_ns))
            report(a.st, kDevErrTimeout, kWhereRescore, 0x80000000u | (uint32_t)round);
        return;
    }
    for (int i = tid; i < kHistBins; i += C::kThreads) {
        const uint32_t v = hist_s[i];
        if (v) atomicAdd(a.hist + (size_t)row * kHistBins + i, v);
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
    k_anchor_score<D><<<grid, C::kThreads, C::kSmemBytes, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_anchor_score(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    return a.d == 128 ? launch_anchor_score_d<128>(a, num_sms, s)
                      : launch_anchor_score_d<64>(a, num_sms, s);
}

template <int D>
static cudaError_t launch_refine_rescore_d(const ScoreArgs &a, cudaStream_t s) {
    using C = RescoreCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(k_refine_rescore<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((a.kappa + C::kEntries - 1) / C::kEntries), (unsigned)(a.B * a.Hkv));
    k_refine_rescore<D><<<grid, C::kThreads, C::kSmemBytes, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_refine_rescore(const ScoreArgs &a, cudaStream_t s) {
    return a.d == 128 ? launch_refine_rescore_d<128>(a, s) : launch_refine_rescore_d<64>(a, s);
}

}  // namespace prism
