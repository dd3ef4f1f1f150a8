// score_max.cu -- full-cache scoring with the group maximum of Eq. (9) of
// "Prism Attention" (section 4.2), on the bf16 key cache:
//   s(i) = scale * max_{j in G(h)} <q_j, k_i>.
// The maximum does not re-associate into one query, so every key row needs
// the G dot products of its group: a [128 x d] x [d x G] product per tile of
// 128 key rows, which runs on the tensor cores (tcgen05.mma, bf16 in, fp32
// accumulate in tensor memory) while the kernel stays bound by the key
// stream.
//
// Persistent grid, one CTA per SM, over the same contiguous tile ranges as the
// group-sum scan (tiles.cuh).  Warp roles:
//   warp 0    TMA producer: per tile, two (d = 128) or one 128-row x 64-column
//             boxes of the key cache with 128-byte swizzle into a 3-stage
//             ring; when the tile's row differs from the stage's last one,
//             the lanes first write the group's queries (B operand, 16 rows:
//             the G heads, repeated to fill 16) in the same swizzled layout;
//   warp 1    allocates 32 tensor-memory columns; one thread issues d/16 MMAs
//             (M = 128 key rows, N = 16, K = 16) per tile into one of two
//             16-column accumulators and commits them to the stage's and the
//             accumulator's mbarriers;
//   warps 2-5 epilogue: each reads its 32-lane quarter of the accumulator
//             (one key row a thread, 16 head columns), takes the maximum,
//             scales, stores the score and counts its first radix digit.
// Every wait is bounded; a timed-out role records the error and stops, and
// the teardown waits (bounded) for the tensor core before freeing tensor
// memory.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_sm100.cuh"
#include "tiles.cuh"

namespace prism {

template <int D>
struct MaxCfg {
    static constexpr int kTileRows = 128;
    // Three stages keep the CTA at ~118 KB of shared memory, so that a CTA of
    // the selection kernel (~107 KB) fits on the same SM: the selections of
    // one anchor overlap the scan of the next.
    static constexpr int kStages = 3;
    static constexpr int kBoxes = D / 64;                     // 64 bf16 = one 128-byte row
    static constexpr int kBoxBytes = kTileRows * 128;
    static constexpr int kKBytes = kBoxes * kBoxBytes;
    static constexpr int kN = 16;                             // MMA N: the group's heads
    static constexpr int kQBoxBytes = kN * 128;
    static constexpr int kQBytes = kBoxes * kQBoxBytes;
    static constexpr int kStageBytes = kKBytes + kQBytes;     // a multiple of 1024
    static constexpr int kKSteps = D / 16;
    static constexpr int kAccBufs = 2;
    static constexpr int kTmemCols = 32;                      // kAccBufs x kN columns
    static constexpr int kEpiWarps = 4;
    static constexpr int kThreads = 32 * (2 + kEpiWarps);
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 1;
    static constexpr int kQRowOff = kBarOff + kNumBars * 8;
    static constexpr int kTmemSlotOff = kQRowOff + kStages * 4;
    static constexpr int kHistOff = (kTmemSlotOff + 4 + 15) & ~15;
    static constexpr int kScratchOff = kHistOff + kHistBins * 4;
    static constexpr int kSmemBytes = kScratchOff + 64 * 4 + 1024;   // + alignment slack
    static_assert(kStageBytes % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
};

__device__ __forceinline__ void epilogue_sync() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(MaxCfg<D>::kThreads, 1)
k_anchor_score_max(const __grid_constant__ CUtensorMap kmap, ScoreArgs a) {
    using C = MaxCfg<D>;
    constexpr int TILE = C::kTileRows;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint64_t *acc_empty = acc_full + C::kAccBufs;
    uint64_t *done = acc_empty + C::kAccBufs;
    int *q_row = reinterpret_cast<int *>(smem + C::kQRowOff);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kTmemSlotOff);
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(smem + C::kHistOff);
    int *scratch = reinterpret_cast<int *>(smem + C::kScratchOff);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // This CTA's contiguous share of the tile order (block-wide scans).
    long long total;
    TileCursor cur0;
    {
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

    for (int i = tid; i < kHistBins; i += blockDim.x) hist_s[i] = 0;
    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            q_row[s] = -1;
        }
        for (int b = 0; b < C::kAccBufs; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], C::kEpiWarps);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int Hq = a.Hkv * a.G;

    if (warp == 0) {
        // ---------------- producer: queries (when the row changes) and key boxes ----
        const uint64_t pol = l2_evict_first_policy();
        const uint16_t *qb = static_cast<const uint16_t *>(a.q);
        TileCursor c = cur0;
        bool failed = false;
        int issued = 0;
        for (int it = 0; it < ntiles && !failed; ++it) {
            const int s = it % C::kStages;
            const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
            bool ok = lane == 0 ? mbar_wait(&empty[s], ph ^ 1u, a.wait_ns) : true;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) report(a.st, kDevErrTimeout, kWhereScore, 0x10000000u | (uint32_t)it);
                failed = true;
                break;
            }
            uint8_t *stage = smem + s * C::kStageBytes;
            const int row = c.b * a.Hkv + c.h;
            if (q_row[s] != row) {
                // B operand: row n of 16 holds query head n % G of the group;
                // 16-byte chunk c8 of a 128-byte row goes to chunk c8 ^ (n % 8).
                uint8_t *qs = stage + C::kKBytes;
                for (int e = lane; e < C::kN * (D / 8); e += 32) {
                    const int n = e / (D / 8), cc = e % (D / 8);
                    const uint16_t *src =
                        qb + ((size_t)c.b * Hq + (size_t)c.h * a.G + (size_t)(n % a.G)) * D + cc * 8;
                    const uint4 v = *reinterpret_cast<const uint4 *>(src);
                    const int box = cc >> 3, c8 = cc & 7;
                    *reinterpret_cast<uint4 *>(qs + box * C::kQBoxBytes + n * 128 +
                                               ((c8 ^ (n & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) q_row[s] = row;
                __syncwarp();
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], (uint32_t)C::kKBytes);
                const int y = row * a.Lmax + c.j * TILE;
#pragma unroll
                for (int box = 0; box < C::kBoxes; ++box)
                    tma_load_2d(stage + box * C::kBoxBytes, &kmap, box * 64, y, &full[s], pol);
            }
            issued = it + 1;
            next_tile<TILE>(c, a.len, a.B, a.Hkv, a.Lmax);
        }
        // Every issued copy lands before the CTA may exit.
        if (lane == 0) {
            for (int it = max(0, issued - C::kStages); it < issued; ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!mbar_wait(&full[s], ph, a.wait_ns))
                    report(a.st, kDevErrTimeout, kWhereScore, 0x20000000u | (uint32_t)it);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ------------------------------------------------
        constexpr uint32_t idesc = idesc_bf16_f32<128, C::kN>();
        bool failed = false;
        for (int it = 0; it < ntiles && !failed; ++it) {
            const int s = it % C::kStages;
            const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
            const int acc = it % C::kAccBufs;
            const uint32_t aph = (uint32_t)(it / C::kAccBufs) & 1u;
            bool ok = true;
            if (lane == 0) {
                ok = mbar_wait(&full[s], ph, a.wait_ns) && mbar_wait(&acc_empty[acc], aph ^ 1u, a.wait_ns);
                if (!ok) report(a.st, kDevErrTimeout, kWhereScore, 0x30000000u | (uint32_t)it);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                failed = true;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sa = smem_addr(smem + s * C::kStageBytes);
                const uint32_t d_tmem = tmem + (uint32_t)(acc * C::kN);
#pragma unroll
                for (int kk = 0; kk < C::kKSteps; ++kk) {
                    const uint32_t ka = sa + (uint32_t)((kk >> 2) * C::kBoxBytes + (kk & 3) * 32);
                    const uint32_t qa = sa + (uint32_t)(C::kKBytes + (kk >> 2) * C::kQBoxBytes + (kk & 3) * 32);
                    tc_mma_bf16(d_tmem, sw128_kmajor_desc(ka), sw128_kmajor_desc(qa), idesc,
                                kk > 0 ? 1u : 0u);
                }
                tc_commit(&empty[s]);          // the stage is free once these MMAs are done
                tc_commit(&acc_full[acc]);     // the accumulator is ready
            }
            __syncwarp();
        }
        // Everything issued has completed before tensor memory is freed.
        if (lane == 0) {
            tc_commit(done);
            if (!mbar_wait(done, 0u, a.wait_ns))
                report(a.st, kDevErrTimeout, kWhereScore, 0x40000000u);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: maximum over the group, scores, histogram -------
        // Scores and the histogram are written only after the preceding kernel
        // has finished.
        pdl_wait();
        const int quarter = warp & 3;                  // tensor-memory lanes 32*quarter ...
        const int r_in_tile = quarter * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
        TileCursor c = cur0;
        int cur_row = -1;
        bool failed = false;
        for (int it = 0; it < ntiles; ++it) {
            const int acc = it % C::kAccBufs;
            const uint32_t aph = (uint32_t)(it / C::kAccBufs) & 1u;
            const int row = c.b * a.Hkv + c.h;
            if (row != cur_row) {
                if (cur_row >= 0) {
                    epilogue_sync();
                    for (int i = tid - 64; i < kHistBins; i += 128) {
                        const uint32_t v = hist_s[i];
                        if (v) {
                            atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
                            hist_s[i] = 0;
                        }
                    }
                    epilogue_sync();
                }
                cur_row = row;
            }
            if (!failed) {
                bool ok = lane == 0 ? mbar_wait(&acc_full[acc], aph, a.wait_ns) : true;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) report(a.st, kDevErrTimeout, kWhereScore, 0x50000000u | (uint32_t)it);
                    failed = true;
                }
            }
            if (!failed) {
                tc_fence_after();
                uint32_t r[16];
                tmem_ld_32x32b_x16(t_lane + (uint32_t)(acc * C::kN), r);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[acc]);
                float m = __uint_as_float(r[0]);
#pragma unroll
                for (int i = 1; i < 16; ++i) m = fmaxf(m, __uint_as_float(r[i]));
                int L = __ldg(a.len + c.b);
                L = L < 0 ? 0 : (L > a.Lmax ? a.Lmax : L);
                const int pos = c.j * TILE + r_in_tile;
                if (pos < L) {
                    const float sc = m * a.scale;
                    a.S[(size_t)row * a.Lmax + pos] = sc;
                    atomicAdd(&hist_s[score_key(sc) >> (32 - kHistBits)], 1u);
                }
            }
            next_tile<TILE>(c, a.len, a.B, a.Hkv, a.Lmax);
        }
        epilogue_sync();
        if (cur_row >= 0) {
            for (int i = tid - 64; i < kHistBins; i += 128) {
                const uint32_t v = hist_s[i];
                if (v) atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

// The key cache as a 2-D bf16 tensor [B * Hkv * Lmax][d], boxes of 128 rows x
// 64 columns, 128-byte swizzle; rows past the end read as zero.
static cudaError_t key_tensor_map(const ScoreArgs &a, CUtensorMap *map) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)a.d, (cuuint64_t)a.B * a.Hkv * (cuuint64_t)a.Lmax};
    const cuuint64_t strides[1] = {(cuuint64_t)a.d * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.k), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
static cudaError_t launch_anchor_score_max_d(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    using C = MaxCfg<D>;
    CUtensorMap map;
    cudaError_t e = key_tensor_map(a, &map);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_anchor_score_max<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.Hkv;
    const long long max_tiles = rows * ((a.Lmax + C::kTileRows - 1) / C::kTileRows);
    const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
    return launch_kernel(k_anchor_score_max<D>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, s,
                         map, a);
}

cudaError_t launch_anchor_score_max(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    return a.d == 128 ? launch_anchor_score_max_d<128>(a, num_sms, s)
                      : launch_anchor_score_max_d<64>(a, num_sms, s);
}

}  // namespace prism
