// score_q2.cu -- the 2-bit proposal keys of "Prism Attention" (section 4.2):
// the quantizer of Eq. (7)-(8) and the full-cache scan of Eq. (9) on the
// quantized keys (row format and tensor-core scoring in q2_impl.cuh).
//
// k_quantize_keys: one thread per group of kQ2Group elements of a key row,
// for the positions [start, len[b]) of every (batch, KV head): alpha =
// (max - min) / 3, beta = min, code = clip(round half up((k - beta) / alpha),
// 0, 3), each an IEEE binary32 operation (no contraction), alpha = 0 -> code 0.
//
// k_anchor_score_q2: the persistent scan of k_anchor_score over 512-row tiles
// of the quantized cache (d/2 bytes a row: 32 KB tiles at d = 128), a 4-stage
// ring of 1-D bulk copies, sixteen consumer warps of 32 rows each scoring on
// the tensor cores, scores and the first-digit histogram as in the bf16 scan.
#include "q2_impl.cuh"
#include "tiles.cuh"

namespace prism {

template <int D>
__global__ void __launch_bounds__(256)
k_quantize_keys(const uint16_t *k, const int32_t *len, int B, int Hkv, int Lmax, int start,
                uint8_t *kq, DevStatus *st) {
    constexpr int M = D / kQ2Group;
    constexpr int RB = q2_row_bytes(D);
    constexpr int KS = D / 16;
    const long long gidx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long rows = (long long)B * Hkv * Lmax;
    if (gidx >= rows * M) return;
    const long long rr = gidx / M;                  // key row of the cache
    const int m = (int)(gidx % M);
    const int b = (int)(rr / ((long long)Hkv * Lmax));
    const int pos = (int)(rr % Lmax);
    int L = __ldg(len + b);
    if (L < 0 || L > Lmax) {
        if (pos == 0 && m == 0) report(st, kDevErrBadLen, kWhereScore, (uint32_t)L);
        L = L < 0 ? 0 : Lmax;
    }
    if (pos < start || pos >= L) return;
    const uint16_t *src = k + rr * D + m * kQ2Group;
    float x[kQ2Group];
#pragma unroll
    for (int e = 0; e < kQ2Group; e += 8) {
        const uint4 v = *reinterpret_cast<const uint4 *>(src + e);
        x[e + 0] = bf16_lo(v.x); x[e + 1] = bf16_hi(v.x);
        x[e + 2] = bf16_lo(v.y); x[e + 3] = bf16_hi(v.y);
        x[e + 4] = bf16_lo(v.z); x[e + 5] = bf16_hi(v.z);
        x[e + 6] = bf16_lo(v.w); x[e + 7] = bf16_hi(v.w);
    }
    float lo = x[0], hi = x[0];
#pragma unroll
    for (int e = 1; e < kQ2Group; ++e) {
        lo = fminf(lo, x[e]);
        hi = fmaxf(hi, x[e]);
    }
    const float a = __fdiv_rn(__fsub_rn(hi, lo), 3.0f);
    uint8_t *row = kq + rr * RB;
    // codes of the group's two k steps (2m, 2m + 1), byte t * KS + kk per lane t
#pragma unroll
    for (int h2 = 0; h2 < kQ2Group / 16; ++h2) {
        const int kk = m * (kQ2Group / 16) + h2;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint32_t byte = 0;
            const int el[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t c = 0;
                if (a > 0.f) {
                    const float y = __fdiv_rn(__fsub_rn(x[16 * h2 + el[i]], lo), a);
                    const float r = floorf(__fadd_rn(y, 0.5f));
                    c = r < 0.f ? 0u : (r > 3.f ? 3u : (uint32_t)r);
                }
                byte |= c << (2 * i);
            }
            row[t * KS + kk] = (uint8_t)byte;
        }
    }
    float *par = reinterpret_cast<float *>(row + D / 4) + 2 * m;
    par[0] = a;
    par[1] = lo;
}

cudaError_t launch_quantize_keys(const void *k, const int32_t *len, int B, int Hkv, int d, int Lmax,
                                 int start, void *kq, DevStatus *st, cudaStream_t s) {
    const long long work = (long long)B * Hkv * Lmax * (d / kQ2Group);
    const int blocks = (int)((work + 255) / 256);
    const uint16_t *kk = static_cast<const uint16_t *>(k);
    uint8_t *out = static_cast<uint8_t *>(kq);
    return d == 128 ? launch_kernel(k_quantize_keys<128>, dim3(blocks), dim3(256), 0, s, kk, len, B,
                                    Hkv, Lmax, start, out, st)
                    : launch_kernel(k_quantize_keys<64>, dim3(blocks), dim3(256), 0, s, kk, len, B,
                                    Hkv, Lmax, start, out, st);
}

template <int D>
struct Q2ScanCfg {
    // 512-row tiles (32 KB at d = 128): each of 16 consumer warps scores 32
    // rows, two 16-row blocks side by side, so that the latency of the mma
    // chains is hidden behind other blocks and warps.
    static constexpr int kTileRows = 512;
    static constexpr int kStages = 4;
    static constexpr int kConsumerWarps = 16;
    static constexpr int kRowsPerWarp = kTileRows / kConsumerWarps;
    static constexpr int kThreads = 32 * (kConsumerWarps + 1);
    static constexpr int kRowBytes = q2_row_bytes(D);
    static constexpr int kTileBytes = kTileRows * kRowBytes;
    static constexpr int kSmemBytes = kStages * kTileBytes + 2 * kStages * 8 + kHistBins * 4 + 64 * 4;
};

__device__ __forceinline__ void q2_consumer_sync() {
    asm volatile("bar.sync 1, 512;" ::: "memory");
}

template <int D, int NT>
__global__ void __launch_bounds__(Q2ScanCfg<D>::kThreads, 1)
k_anchor_score_q2(ScoreArgs a) {
    using C = Q2ScanCfg<D>;
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

    if (warp == C::kConsumerWarps) {
        // ---------------- producer: one thread issues the bulk copies -------------
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            const uint8_t *kb = static_cast<const uint8_t *>(a.k);
            TileCursor c = cur0;
            bool failed = false;
            int issued = 0;
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!failed && !mbar_wait(&empty[s], ph ^ 1u, a.wait_ns)) {
                    report(a.st, kDevErrTimeout, kWhereScore, 0x60000000u | (uint32_t)it);
                    failed = true;
                }
                if (!failed) {
                    int L = __ldg(a.len + c.b);
                    L = L < 0 ? 0 : (L > a.Lmax ? a.Lmax : L);
                    const int rows = min(TILE, L - c.j * TILE);
                    const uint32_t bytes = (uint32_t)rows * C::kRowBytes;
                    const size_t off = ((size_t)(c.b * a.Hkv + c.h) * a.Lmax + (size_t)c.j * TILE) *
                                       C::kRowBytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_load(stages + s * C::kTileBytes, kb + off, bytes, &full[s], pol);
                    issued = it + 1;
                }
                next_tile<TILE>(c, a.len, a.B, a.Hkv, a.Lmax);
            }
            for (int it = max(0, issued - C::kStages); it < issued; ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
                if (!mbar_wait(&full[s], ph, a.wait_ns))
                    report(a.st, kDevErrTimeout, kWhereScore, 0x70000000u | (uint32_t)it);
            }
        }
        return;
    }

    // ---------------- consumers: 16 rows per warp --------------------------------
    pdl_wait();
    const uint16_t *qb = static_cast<const uint16_t *>(a.q);
    const int Hq = a.Hkv * a.G;
    Q2Query<D, NT> Q;
    int cur_row = -1;
    TileCursor c = cur0;
    bool failed = false;
    const int g = lane >> 2, t = lane & 3;
    for (int it = 0; it < ntiles; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (uint32_t)(it / C::kStages) & 1u;
        const int row = c.b * a.Hkv + c.h;
        if (row != cur_row) {
            if (cur_row >= 0) {
                q2_consumer_sync();
                for (int i = tid; i < kHistBins; i += 32 * C::kConsumerWarps) {
                    const uint32_t v = hist_s[i];
                    if (v) {
                        atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
                        hist_s[i] = 0;
                    }
                }
                q2_consumer_sync();
            }
            q2_load_query<D, NT>(Q, qb + ((size_t)c.b * Hq + (size_t)c.h * a.G) * D, a.G, lane);
            cur_row = row;
        }
        int L = __ldg(a.len + c.b);
        L = L < 0 ? 0 : (L > a.Lmax ? a.Lmax : L);
        if (!failed && !mbar_wait(&full[s], ph, a.wait_ns)) {
            report(a.st, kDevErrTimeout, kWhereScore, 0x50000000u | (uint32_t)it);
            failed = true;
        }
        if (!failed) {
            const uint8_t *rows_w = stages + s * C::kTileBytes + warp * C::kRowsPerWarp * C::kRowBytes;
            float2 mx[C::kRowsPerWarp / 32][2];
#pragma unroll
            for (int pr = 0; pr < C::kRowsPerWarp / 32; ++pr)
                q2_group_max_rows<D, NT, 2>(rows_w + pr * 32 * C::kRowBytes, 16 * C::kRowBytes, Q,
                                            lane, mx[pr]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (t < 2) {
#pragma unroll
                for (int blk = 0; blk < C::kRowsPerWarp / 16; ++blk) {
                    const float2 m2 = mx[blk >> 1][blk & 1];
                    const int pos = c.j * TILE + warp * C::kRowsPerWarp + 16 * blk + g + (t == 1 ? 8 : 0);
                    if (pos < L) {
                        const float sc = (t == 1 ? m2.y : m2.x) * a.scale;
                        a.S[(size_t)row * a.Lmax + pos] = sc;
                        atomicAdd(&hist_s[score_key(sc) >> (32 - kHistBits)], 1u);
                    }
                }
            }
        }
        next_tile<TILE>(c, a.len, a.B, a.Hkv, a.Lmax);
    }
    q2_consumer_sync();
    pdl_launch_dependents();
    if (cur_row >= 0) {
        for (int i = tid; i < kHistBins; i += 32 * C::kConsumerWarps) {
            const uint32_t v = hist_s[i];
            if (v) atomicAdd(a.hist + (size_t)cur_row * kHistBins + i, v);
        }
    }
}

template <int D, int NT>
static cudaError_t launch_anchor_score_q2_d(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    using C = Q2ScanCfg<D>;
    cudaError_t e = cudaFuncSetAttribute(k_anchor_score_q2<D, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.Hkv;
    const long long max_tiles = rows * ((a.Lmax + C::kTileRows - 1) / C::kTileRows);
    const int grid = (int)(max_tiles < num_sms ? max_tiles : num_sms);
    return launch_kernel(k_anchor_score_q2<D, NT>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, s,
                         a);
}

cudaError_t launch_anchor_score_q2(const ScoreArgs &a, int num_sms, cudaStream_t s) {
    if (a.G > 8)
        return a.d == 128 ? launch_anchor_score_q2_d<128, 2>(a, num_sms, s)
                          : launch_anchor_score_q2_d<64, 2>(a, num_sms, s);
    return a.d == 128 ? launch_anchor_score_q2_d<128, 1>(a, num_sms, s)
                      : launch_anchor_score_q2_d<64, 1>(a, num_sms, s);
}

}  // namespace prism
