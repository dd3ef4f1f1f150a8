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
// (Eq. (5)): rows are gathered with 16-byte non-caching loads.
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
// Refined layer: score only the proposal positions (Eq. (5)).
template <int D>
struct RescoreCfg {
    static constexpr int kTile = 128;        // proposal slots per CTA
    static constexpr int kWarps = 8;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kNL = D / 8;
    static constexpr int kRPI = 32 / kNL;
    static constexpr int kRowsPerWarp = kTile / kWarps;
    static constexpr int kSteps = kRowsPerWarp / kRPI;
};

template <int D>
__global__ void __launch_bounds__(RescoreCfg<D>::kThreads)
k_refine_rescore(ScoreArgs a) {
    using C = RescoreCfg<D>;
    __shared__ uint32_t hist_s[kHistBins];
    const int row = blockIdx.y;
    const int n = a.ctl[row].n_prop;
    const int e0 = blockIdx.x * C::kTile;
    if (e0 >= n) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int slice = lane % C::kNL, sub = lane / C::kNL;
    const int Hq = a.Hkv * a.G;

    for (int i = tid; i < kHistBins; i += C::kThreads) hist_s[i] = 0;

    const int32_t *cpos = a.cpos + (size_t)row * a.Lmax;
    const uint16_t *kb = static_cast<const uint16_t *>(a.k) +
                                  (size_t)row * a.Lmax * D;
    uint4 kv[C::kSteps];
    const int ebase = e0 + warp * C::kRowsPerWarp + sub;
#pragma unroll
    for (int st = 0; st < C::kSteps; ++st) {
        const int e = ebase + st * C::kRPI;
        if (e < n) {
            const int p = __ldg(cpos + e);
            kv[st] = ld_nc_v4(kb + (size_t)p * D + slice * 8);
        } else {
            kv[st] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    float qreg[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qreg[e] = 0.f;
    const uint16_t *qb = static_cast<const uint16_t *>(a.q);
    for (int g = 0; g < a.G; ++g) {
        const uint4 w = *reinterpret_cast<const uint4 *>(
            qb + ((size_t)b * Hq + (size_t)h * a.G + g) * D + slice * 8);
        qreg[0] += bf16_lo(w.x); qreg[1] += bf16_hi(w.x);
        qreg[2] += bf16_lo(w.y); qreg[3] += bf16_hi(w.y);
        qreg[4] += bf16_lo(w.z); qreg[5] += bf16_hi(w.z);
        qreg[6] += bf16_lo(w.w); qreg[7] += bf16_hi(w.w);
    }
    float part[C::kSteps];
#pragma unroll
    for (int st = 0; st < C::kSteps; ++st) part[st] = dot8(kv[st], qreg);
    transpose_reduce<C::kSteps, C::kNL>(part, lane);
    __syncthreads();   // hist_s zeroed
    const int item = transpose_item<C::kSteps, C::kNL>(lane);
    const int e = ebase + item * C::kRPI;
    if (transpose_writer<C::kSteps, C::kNL>(lane) && e < n) {
        const float sc = part[0] * a.scale;
        a.S[(size_t)row * a.Lmax + e] = sc;
        atomicAdd(&hist_s[score_key(sc) >> (32 - kHistBits)], 1u);
    }
    __syncthreads();
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
static cudaError_t launch_refine_rescore_d(const ScoreArgs &a, long long max_prop,
                                           cudaStream_t s) {
    using C = RescoreCfg<D>;
    const long long tiles = (max_prop + C::kTile - 1) / C::kTile;
    if (tiles <= 0) return cudaSuccess;
    dim3 grid((unsigned)tiles, (unsigned)(a.B * a.Hkv));
    k_refine_rescore<D><<<grid, C::kThreads, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_refine_rescore(const ScoreArgs &a, long long max_prop, cudaStream_t s) {
    return a.d == 128 ? launch_refine_rescore_d<128>(a, max_prop, s)
                      : launch_refine_rescore_d<64>(a, max_prop, s);
}

}  // namespace prism
