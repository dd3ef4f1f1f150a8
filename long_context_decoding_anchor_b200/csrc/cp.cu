// cp.cu -- helper kernels of the context-parallel decode step (prism_cp.h).
//
// One rank holds the positions [lo, lo + cap) of every sequence.  It runs the
// single-GPU kernels (scoring, rescoring, selection, attention) on its shard
// in local positions; these kernels adapt their inputs and outputs:
//  - k_cp_prepare: the shard lengths, and the refined layer's proposal
//    ("Prism Attention", Eq. (5): every position within r of a source token,
//    clipped to [0, len)) restricted to the shard, as a radius-0 source; or a
//    global selection in local positions for the attention.
//  - k_cp_pack: a local selection as (global position, score) pairs (the
//    rescoring of a refined layer leaves its candidates' scores by position).
//  - k_cp_merge_compact / k_cp_merge_hist: the gathered pairs of all ranks as
//    one candidate list per row, for the exact selection (the top-k of a
//    union is the top-k of the union of the parts' top-k).
//  - k_cp_reduce / k_cp_combine: split softmax across ranks,
//    o = sum_r e^(m_r - M) acc_r / sum_r e^(m_r - M) l_r.
#include <cuda_bf16.h>

#include "cp_internal.cuh"

namespace prism {

constexpr int kCpThreads = 256;
constexpr int kCpSplit = 8;          // CTAs per row of k_cp_prepare

// Grid (rows, kCpSplit).  For a proposal, every CTA of a row counts the
// positions of all entries (one run of entries per thread, a block scan) and
// writes the positions of its own share of the output slots.
__global__ void __launch_bounds__(kCpThreads)
k_cp_prepare(CpPrepArgs a) {
    __shared__ int scratch[40];
    const int row = blockIdx.x, part = blockIdx.y;
    const int b = row / a.Hkv, h = row % a.Hkv;
    const int tid = threadIdx.x;
    pdl_wait();
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereCanon);
    const int n_loc = max(0, min(L - a.lo, a.cap));
    if (h == 0 && part == 0 && tid == 0) a.llen[b] = n_loc;
    if (a.what == kCpPrepLen) return;
    const int32_t *src = a.src + (size_t)row * a.src_kappa;
    int32_t *out = a.out + (size_t)row * a.out_kappa;
    if (a.what == kCpPrepSelection) {
        for (int t = part * kCpThreads + tid; t < a.src_kappa; t += kCpSplit * kCpThreads) {
            const int p = __ldg(src + t);
            out[t] = (p >= a.lo && p < a.lo + n_loc) ? p - a.lo : -1;
        }
        return;
    }
    // The proposal inside the shard: entry j owns the positions of its window
    // that no earlier entry's window covers (owned_range), here cut to the
    // shard [lo, lo + n_loc).
    const int per = (a.src_kappa + kCpThreads - 1) / kCpThreads;
    const int j0 = min(a.src_kappa, tid * per), j1 = min(a.src_kappa, j0 + per);
    const long long shard_hi = (long long)a.lo + n_loc - 1;
    int cnt = 0;
    for (int j = j0; j < j1; ++j) {
        int lo_j = 0;
        const int own = owned_range(src, j, a.radius, L, &lo_j, part == 0 ? a.st : nullptr,
                                    kWhereCanon);
        const long long s = max((long long)lo_j, (long long)a.lo);
        const long long e = min((long long)lo_j + own - 1, shard_hi);
        if (own > 0 && e >= s) cnt += (int)(e - s + 1);
    }
    int total;
    int at = block_exclusive_scan(cnt, scratch, &total);
    const int cap_total = min(total, a.out_kappa);
    const int o_begin = (int)((long long)part * cap_total / kCpSplit);
    const int o_end = (int)((long long)(part + 1) * cap_total / kCpSplit);
    for (int j = j0; j < j1 && at < o_end; ++j) {
        int lo_j = 0;
        const int own = owned_range(src, j, a.radius, L, &lo_j, nullptr, kWhereCanon);
        const long long s = max((long long)lo_j, (long long)a.lo);
        const long long e = min((long long)lo_j + own - 1, shard_hi);
        if (own <= 0 || e < s) continue;
        const int len = (int)(e - s + 1);
        // this entry's slots [at, at + len) within this CTA's [o_begin, o_end)
        const int t0 = max(at, o_begin), t1 = min(at + len, o_end);
        for (int t = t0; t < t1; ++t) out[t] = (int)(s - a.lo) + (t - at);
        at += len;
    }
    // the rest of the source is padding
    for (int t = cap_total + part * kCpThreads + tid; t < a.out_kappa; t += kCpSplit * kCpThreads)
        out[t] = -1;
    if (part == 0 && tid == 0 && total > a.out_kappa)
        report(a.st, kDevErrInternal, kWhereCanon, (uint32_t)total);
}

cudaError_t launch_cp_prepare(const CpPrepArgs &a, cudaStream_t s) {
    return launch_kernel(k_cp_prepare, dim3(a.B * a.Hkv, kCpSplit), dim3(kCpThreads), 0, s, a);
}

__global__ void __launch_bounds__(kCpThreads)
k_cp_pack(CpPackArgs a) {
    const int row = blockIdx.x;
    pdl_wait();
    const int32_t *sel = a.sel + (size_t)row * a.n;
    const float *S = a.S + (size_t)row * a.sstride;
    for (int t = threadIdx.x; t < a.n; t += kCpThreads) {
        const int i = __ldcg(sel + t);
        const bool ok = i >= 0 && i < a.sstride;
        a.pos_out[(size_t)row * a.n + t] = ok ? a.lo + i : -1;
        a.score_out[(size_t)row * a.n + t] = ok ? __ldcg(S + i) : -INFINITY;
    }
}

cudaError_t launch_cp_pack(const CpPackArgs &a, cudaStream_t s) {
    return launch_kernel(k_cp_pack, dim3(a.rows), dim3(kCpThreads), 0, s, a);
}

// The rows of the R lists are consecutive shards, so keeping the valid
// entries in rank order keeps the positions ascending.
constexpr int kMergeThreads = 1024;

__global__ void __launch_bounds__(kMergeThreads)
k_cp_merge_compact(CpMergeArgs a) {
    __shared__ int scratch[40];
    const int row = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_wait();
    const int L = load_len(a.len, row / a.Hkv, a.Lmax, a.st, kWhereCollect);
    const int items = a.R * a.n;
    float *S = a.S + (size_t)row * a.cstride;
    int32_t *cpos = a.cpos + (size_t)row * a.cstride;
    int base = 0;
    for (int i0 = 0; i0 < items; i0 += kMergeThreads) {
        const int i = i0 + tid;
        int p = -1;
        float sc = 0.f;
        if (i < items) {
            const size_t at = ((size_t)(i / a.n) * a.rows + row) * a.n + (i % a.n);
            p = __ldg(a.pos + at);
            sc = __ldg(a.score + at);
            if (p >= L) {
                report(a.st, kDevErrBadIndex, kWhereCollect, (uint32_t)p);
                p = -1;
            }
        }
        int total;
        const int excl = block_exclusive_scan(p >= 0 ? 1 : 0, scratch, &total);
        if (p >= 0) {
            S[base + excl] = sc;
            cpos[base + excl] = p;
        }
        base += total;
    }
    __syncthreads();
    for (int i = tid + 1; i < base; i += kMergeThreads)
        if (cpos[i - 1] >= cpos[i]) report(a.st, kDevErrBadIndex, kWhereCollect, (uint32_t)cpos[i]);
    if (tid == 0) a.count_out[(size_t)row * (items + 1) + items] = base;
}

__global__ void __launch_bounds__(512)
k_cp_merge_hist(CpMergeArgs a) {
    __shared__ uint32_t h[kHistBins];
    const int row = blockIdx.x;
    const int items = a.R * a.n;
    for (int i = threadIdx.x; i < kHistBins; i += 512) h[i] = 0;
    __syncthreads();
    pdl_wait();
    const int n = __ldcg(a.count_out + (size_t)row * (items + 1) + items);
    const float *S = a.S + (size_t)row * a.cstride;
    for (int i = threadIdx.x; i < n; i += 512)
        atomicAdd(&h[score_key(__ldcg(S + i)) >> (32 - kHistBits)], 1u);
    __syncthreads();
    for (int i = threadIdx.x; i < kHistBins; i += 512) a.hist[(size_t)row * kHistBins + i] = h[i];
}

cudaError_t launch_cp_merge_prepare(const CpMergeArgs &a, cudaStream_t s) {
    cudaError_t e = launch_kernel(k_cp_merge_compact, dim3(a.rows), dim3(kMergeThreads), 0, s, a);
    if (e != cudaSuccess) return e;
    return launch_kernel(k_cp_merge_hist, dim3(a.rows), dim3(512), 0, s, a);
}

// One CTA per (row, query head); thread c owns column c of the accumulator.
__global__ void __launch_bounds__(128)
k_cp_reduce(CpReduceArgs a) {
    __shared__ float wts[kAttnChunk * 4];
    __shared__ float stat[2];
    const int row = blockIdx.x, g = blockIdx.y;
    const int tid = threadIdx.x;
    pdl_wait();
    const float *pm = a.part_ml + (size_t)row * a.nsplit * a.G * 2;
    if (tid < 32) {
        float M = -INFINITY;
        for (int s = tid; s < a.nsplit; s += 32) M = fmaxf(M, __ldcg(pm + ((size_t)s * a.G + g) * 2));
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float den = 0.f;
        for (int s = tid; s < a.nsplit; s += 32) {
            const float m = __ldcg(pm + ((size_t)s * a.G + g) * 2);
            const float w = (M == -INFINITY || m == -INFINITY) ? 0.f : __expf(m - M);
            den = fmaf(w, __ldcg(pm + ((size_t)s * a.G + g) * 2 + 1), den);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        if (tid == 0) {
            stat[0] = M;
            stat[1] = den;
        }
    }
    __syncthreads();
    const float M = stat[0];
    float *out = a.out + ((size_t)row * a.G + g) * (a.d + 2);
    for (int s0 = 0; s0 < a.nsplit; s0 += kAttnChunk * 4) {
        const int cnt = min(kAttnChunk * 4, a.nsplit - s0);
        __syncthreads();
        for (int s = tid; s < cnt; s += 128) {
            const float m = __ldcg(pm + ((size_t)(s0 + s) * a.G + g) * 2);
            wts[s] = (M == -INFINITY || m == -INFINITY) ? 0.f : __expf(m - M);
        }
        __syncthreads();
        if (tid < a.d) {
            float acc = s0 == 0 ? 0.f : out[tid];
            for (int s = 0; s < cnt; ++s) {
                const float w = wts[s];
                if (w != 0.f)
                    acc = fmaf(w, __ldcg(a.part_acc + (((size_t)row * a.nsplit + s0 + s) * a.G + g) * a.d + tid), acc);
            }
            out[tid] = acc;
        }
    }
    if (tid == 0) {
        out[a.d] = M;
        out[a.d + 1] = stat[1];
    }
}

cudaError_t launch_cp_reduce(const CpReduceArgs &a, cudaStream_t s) {
    return launch_kernel(k_cp_reduce, dim3(a.rows, a.G), dim3(128), 0, s, a);
}

// One CTA per query head; thread c owns column c.
__global__ void __launch_bounds__(128)
k_cp_combine(CpCombineArgs a) {
    const int hd = blockIdx.x;
    const int tid = threadIdx.x;
    pdl_wait();
    const size_t stride = (size_t)a.heads * (a.d + 2);
    const float *p0 = a.part + (size_t)hd * (a.d + 2);
    float M = -INFINITY;
    for (int r = 0; r < a.R; ++r) M = fmaxf(M, __ldg(p0 + r * stride + a.d));
    if (tid >= a.d) return;
    float num = 0.f, den = 0.f;
    if (M != -INFINITY) {
        for (int r = 0; r < a.R; ++r) {
            const float *p = p0 + r * stride;
            const float m = __ldg(p + a.d);
            if (m == -INFINITY) continue;
            const float w = __expf(m - M);
            num = fmaf(w, __ldg(p + tid), num);
            den = fmaf(w, __ldg(p + a.d + 1), den);
        }
    }
    const float o = den > 0.f ? num / den : 0.f;
    static_cast<__nv_bfloat16 *>(a.out)[(size_t)hd * a.d + tid] = __float2bfloat16_rn(o);
}

cudaError_t launch_cp_combine(const CpCombineArgs &a, cudaStream_t s) {
    return launch_kernel(k_cp_combine, dim3(a.heads), dim3(128), 0, s, a);
}

}  // namespace prism
