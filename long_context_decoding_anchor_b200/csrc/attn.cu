// attn.cu -- sparse GQA decode attention over a selection (the SparseAttn
// step of Algorithm 1 in "Prism Attention").
//
// For KV head h and each query head j of its group:
//   z_i = scale * <q_j, k_i>, i in T;   o_j = sum_i softmax(z)_i v_i.
// Split-K: one CTA per (64-slot chunk of T, (batch, KV head)) gathers its K
// and V rows once for all G query heads with 16-byte cp.async copies into
// shared memory (rows of padding slots are zero-filled, not read), forms the
// G x 64 logits, and writes an unnormalised partial (running max m, sum l,
// accumulator acc[d]) per query head.  The last CTA of a row to finish merges
// the row's partials with the usual rescaling by exp(m_s - M).
#include <cuda_bf16.h>

#include "prism_internal.cuh"

namespace prism {

template <int D, int G>
struct AttnCfg {
    static constexpr int kC = kAttnChunk;
    static constexpr int kThreads = 128;
    static constexpr int kWarps = kThreads / 32;
    static constexpr int kNL = D / 8;
    static constexpr int kRPI = 32 / kNL;
    static constexpr int kRowsPerWarp = kC / kWarps;
    static constexpr int kSteps = kRowsPerWarp / kRPI;
    static constexpr int kPairs = G * kNL;                         // (head, 8-element slice)
    static constexpr int kTPR = kPairs >= kThreads ? 1 : kThreads / kPairs;   // threads per pair
    static constexpr int kPPT = kPairs >= kThreads ? kPairs / kThreads : 1;   // pairs per thread
    static constexpr int kChunksPerRow = D / 8;
    static_assert(G <= kNL, "group larger than lanes per row");
};

// Merge the split-K partials of one (batch, KV head) row:
//   O_j = sum_s exp(m_s - M) acc_s / sum_s exp(m_s - M) l_s,  M = max_s m_s.
// Every split's (m, l) is read once, by all threads together, into `mlbuf`
// (at least kAttnChunk * G float2: the row's K tile, free by now) when the
// row has at most kAttnChunk splits; `wbuf` (at least G * kAttnChunk floats)
// then caches the split weights.  Longer rows read (m, l) from L2 as they go.
template <int D, int G>
__device__ void combine_row(const AttnArgs &a, int row, int b, int h, int nsplit, float *wbuf,
                            float2 *mlbuf) {
    __shared__ float Mh[G], inv_den[G], den_h[G];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float *pm = a.part_ml + (size_t)row * nsplit * G * 2;
    const bool cache = nsplit <= kAttnChunk;
    constexpr int kC4 = G * D / 4;
    constexpr int kBatch = 16;
    const float4 *pa4 = reinterpret_cast<const float4 *>(a.part_acc + (size_t)row * nsplit * G * D);
    if (cache) {
        const float2 *pm2 = reinterpret_cast<const float2 *>(pm);
        for (int i = tid; i < nsplit * G; i += blockDim.x) mlbuf[i] = __ldcg(pm2 + i);
        __syncthreads();
    }
    auto ml_at = [&](int s, int g) -> float2 {
        return cache ? mlbuf[s * G + g]
                     : make_float2(__ldcg(pm + ((size_t)s * G + g) * 2), __ldcg(pm + ((size_t)s * G + g) * 2 + 1));
    };
    for (int g = warp; g < G; g += 4) {
        float M = -INFINITY;
        for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, ml_at(s, g).x);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float den = 0.f;
        for (int s = lane; s < nsplit; s += 32) {
            const float2 ml = ml_at(s, g);
            const float w = (M == -INFINITY || ml.x == -INFINITY) ? 0.f : __expf(ml.x - M);
            if (cache) wbuf[g * kAttnChunk + s] = w;
            den = fmaf(w, ml.y, den);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        if (lane == 0) {
            Mh[g] = M;
            den_h[g] = den;
            inv_den[g] = den > 0.f ? 1.f / den : 0.f;
        }
    }
    __syncthreads();
    // Each thread owns float4 columns of the [G][D] accumulator; the partials
    // of 16 splits are loaded at a time so their L2 round trips overlap.
    uint16_t *out = static_cast<uint16_t *>(a.out) + ((size_t)b * a.Hkv * G + (size_t)h * G) * D;
    for (int c4 = threadIdx.x; c4 < kC4; c4 += blockDim.x) {
        const int g = (c4 * 4) / D;
        const float Mg = Mh[g];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (Mg != -INFINITY) {
            for (int s0 = 0; s0 < nsplit; s0 += kBatch) {
                float4 v[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u)
                    v[u] = s0 + u < nsplit ? __ldcg(pa4 + (size_t)(s0 + u) * kC4 + c4)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int sp = s0 + u;
                    if (sp >= nsplit) break;
                    float w;
                    if (cache) {
                        w = wbuf[g * kAttnChunk + sp];
                    } else {
                        const float m = __ldcg(pm + ((size_t)sp * G + g) * 2);
                        w = m == -INFINITY ? 0.f : __expf(m - Mg);
                    }
                    acc.x = fmaf(w, v[u].x, acc.x);
                    acc.y = fmaf(w, v[u].y, acc.y);
                    acc.z = fmaf(w, v[u].z, acc.z);
                    acc.w = fmaf(w, v[u].w, acc.w);
                }
            }
        }
        if (a.cp_part) {
            // this rank's partial of the row: the accumulator unnormalised, M, l
            float *cp = a.cp_part + ((size_t)row * G + g) * (D + 2);
            const int c = (c4 * 4) % D;
            cp[c] = acc.x;
            cp[c + 1] = acc.y;
            cp[c + 2] = acc.z;
            cp[c + 3] = acc.w;
            if (c == 0) {
                cp[D] = Mg;
                cp[D + 1] = den_h[g];
            }
            continue;
        }
        const float sc = inv_den[g];
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * sc, acc.y * sc);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * sc, acc.w * sc);
        uint2 packed;
        packed.x = *reinterpret_cast<const uint32_t *>(&lo);
        packed.y = *reinterpret_cast<const uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(out + (size_t)c4 * 4) = packed;
    }
}

template <int D, int G>
__global__ void __launch_bounds__(128)
k_sparse_attn(AttnArgs a) {
    using C = AttnCfg<D, G>;
    __shared__ __align__(16) uint16_t Ks[C::kC * D];
    __shared__ __align__(16) uint16_t Vs[C::kC * D];
    __shared__ float z[G][C::kC];
    __shared__ float ml[G][2];
    __shared__ int idx_s[C::kC];
    __shared__ __align__(16) float red[C::kTPR > 1 ? C::kTPR * C::kPairs * 8 : 1];

    const int chunk = blockIdx.x, row = blockIdx.y;
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereAttn);
    const int t0 = chunk * C::kC;
    // The selection may come from the preceding kernel of this stream, and the
    // partials buffer is shared with the preceding attention kernel.
    pdl_wait();
    pdl_launch_dependents();

    if (tid < C::kC) {
        int i = -1;
        if (t0 + tid < a.n_idx) {
            i = __ldg(a.idx + (size_t)row * a.idx_stride + t0 + tid);
            if (i >= L) {
                report(a.st, kDevErrBadIndex, kWhereAttn, (uint32_t)i);
                i = -1;
            }
            if (i < -1) i = -1;
        }
        idx_s[tid] = i;
    }
    __syncthreads();

    const uint16_t *kbase = static_cast<const uint16_t *>(a.k) + (size_t)row * a.Lmax * D;
    const uint16_t *vbase = static_cast<const uint16_t *>(a.v) + (size_t)row * a.Lmax * D;
    for (int c = tid; c < C::kC * C::kChunksPerRow; c += C::kThreads) {
        const int r = c / C::kChunksPerRow, sl = c % C::kChunksPerRow;
        const int i = idx_s[r];
        const size_t off = (size_t)(i < 0 ? 0 : i) * D + sl * 8;
        cp_async16(&Ks[r * D + sl * 8], kbase + off, i < 0 ? 0u : 16u);
    }
    cp_async_commit();
    for (int c = tid; c < C::kC * C::kChunksPerRow; c += C::kThreads) {
        const int r = c / C::kChunksPerRow, sl = c % C::kChunksPerRow;
        const int i = idx_s[r];
        const size_t off = (size_t)(i < 0 ? 0 : i) * D + sl * 8;
        cp_async16(&Vs[r * D + sl * 8], vbase + off, i < 0 ? 0u : 16u);
    }
    cp_async_commit();

    // Query heads of this group, this lane's 8 elements of each.
    const int slice = lane % C::kNL, sub = lane / C::kNL;
    float qreg[G][8];
    const uint16_t *qb = static_cast<const uint16_t *>(a.q) +
                                  ((size_t)b * a.Hkv * G + (size_t)h * G) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint4 w = *reinterpret_cast<const uint4 *>(qb + (size_t)g * D + slice * 8);
        qreg[g][0] = bf16_lo(w.x); qreg[g][1] = bf16_hi(w.x);
        qreg[g][2] = bf16_lo(w.y); qreg[g][3] = bf16_hi(w.y);
        qreg[g][4] = bf16_lo(w.z); qreg[g][5] = bf16_hi(w.z);
        qreg[g][6] = bf16_lo(w.w); qreg[g][7] = bf16_hi(w.w);
    }

    cp_async_wait<1>();
    __syncthreads();

    // Logits.
#pragma unroll
    for (int st = 0; st < C::kSteps; ++st) {
        const int r = warp * C::kRowsPerWarp + st * C::kRPI + sub;
        const uint4 kv = *reinterpret_cast<const uint4 *>(&Ks[r * D + slice * 8]);
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part[g] = dot8(kv, qreg[g]);
        transpose_reduce<G, C::kNL>(part, lane);
        if (transpose_writer<G, C::kNL>(lane)) {
            const int g = transpose_item<G, C::kNL>(lane);
            z[g][r] = idx_s[r] >= 0 ? part[0] * a.scale : -INFINITY;
        }
    }
    __syncthreads();

    // Per-head chunk softmax statistics; z becomes exp(z - m).
    for (int g = warp; g < G; g += C::kWarps) {
        float v0 = z[g][lane], v1 = z[g][lane + 32];
        float m = fmaxf(v0, v1);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float p0 = 0.f, p1 = 0.f;
        if (m != -INFINITY) {
            p0 = __expf(v0 - m);
            p1 = __expf(v1 - m);
        }
        float l = p0 + p1;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        z[g][lane] = p0;
        z[g][lane + 32] = p1;
        if (lane == 0) {
            ml[g][0] = m;
            ml[g][1] = l;
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // Weighted V accumulation: thread -> (head, 8-element slice) pair(s).
    const size_t pbase = ((size_t)row * gridDim.x + chunk) * G;
#pragma unroll
    for (int pp = 0; pp < C::kPPT; ++pp) {
        const int pair = (C::kTPR > 1) ? (tid % C::kPairs) : (tid + pp * C::kThreads);
        const int part_id = (C::kTPR > 1) ? (tid / C::kPairs) : 0;
        const int g = pair / C::kNL, sl = pair % C::kNL;
        constexpr int kRowsPer = C::kC / C::kTPR;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        const int r0 = part_id * kRowsPer;
#pragma unroll 4
        for (int r = r0; r < r0 + kRowsPer; ++r) {
            const float p = z[g][r];
            const uint4 vv = *reinterpret_cast<const uint4 *>(&Vs[r * D + sl * 8]);
            acc[0] = fmaf(p, bf16_lo(vv.x), acc[0]); acc[1] = fmaf(p, bf16_hi(vv.x), acc[1]);
            acc[2] = fmaf(p, bf16_lo(vv.y), acc[2]); acc[3] = fmaf(p, bf16_hi(vv.y), acc[3]);
            acc[4] = fmaf(p, bf16_lo(vv.z), acc[4]); acc[5] = fmaf(p, bf16_hi(vv.z), acc[5]);
            acc[6] = fmaf(p, bf16_lo(vv.w), acc[6]); acc[7] = fmaf(p, bf16_hi(vv.w), acc[7]);
        }
        if (C::kTPR > 1) {
            float *dst = red + ((size_t)part_id * C::kPairs + pair) * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = acc[e];
            __syncthreads();
            if (part_id == 0) {
                for (int q = 1; q < C::kTPR; ++q) {
                    const float *src = red + ((size_t)q * C::kPairs + pair) * 8;
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[e] += src[e];
                }
            }
        }
        if (part_id == 0) {
            float4 *o = reinterpret_cast<float4 *>(a.part_acc + (pbase + g) * D + sl * 8);
            o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    }
    if (tid < G) {
        a.part_ml[(pbase + tid) * 2 + 0] = ml[tid][0];
        a.part_ml[(pbase + tid) * 2 + 1] = ml[tid][1];
    }

    // The last CTA of the row to finish merges the partials (no waiting: an
    // atomic counter decides which CTA that is).
    __shared__ int is_last;
    __syncthreads();
    if (tid == 0) {
        // the block's partials (ordered before this thread by the barrier)
        // become visible before the count: the fence is cumulative
        __threadfence();
        is_last = atomicAdd(&a.ctl[row].done_attn, 1u) == gridDim.x - 1;
        if (is_last) __threadfence();
    }
    __syncthreads();
    if (!is_last) return;
    combine_row<D, G>(a, row, b, h, gridDim.x, &z[0][0], reinterpret_cast<float2 *>(Ks));
    if (tid == 0) a.ctl[row].done_attn = 0;
}

template <int D, int G>
static cudaError_t launch_attn_dg(const AttnArgs &a, cudaStream_t s) {
    const int rows = a.B * a.Hkv;
    const int nsplit = (a.n_idx + kAttnChunk - 1) / kAttnChunk;
    return launch_kernel(k_sparse_attn<D, G>, dim3(nsplit, rows), dim3(128), 0, s, a);
}

template <int D>
static cudaError_t launch_attn_d(const AttnArgs &a, cudaStream_t s) {
    switch (a.G) {
        case 1: return launch_attn_dg<D, 1>(a, s);
        case 2: return launch_attn_dg<D, 2>(a, s);
        case 4: return launch_attn_dg<D, 4>(a, s);
        case 8: return launch_attn_dg<D, 8>(a, s);
        default: break;
    }
    if constexpr (D == 128) {
        if (a.G == 16) return launch_attn_dg<D, 16>(a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t s) {
    return a.d == 128 ? launch_attn_d<128>(a, s) : launch_attn_d<64>(a, s);
}

}  // namespace prism
