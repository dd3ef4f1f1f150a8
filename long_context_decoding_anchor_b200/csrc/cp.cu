// cp.cu -- helper kernels of the context-parallel decode step (prism_cp.h).
//
// One rank holds the positions [lo, lo + cap) of every sequence.  It runs the
// single-GPU kernels (scoring, rescoring, selection, attention) on its shard
// in local positions; these kernels adapt their inputs and outputs:
//  - k_cp_prepare: the shard lengths, and a global selection in local
//    positions for the attention.  (A refined layer's rescoring cuts the
//    proposal of the global source to the shard itself.)
//  - k_cp_pack: a local selection as (global position, score) pairs (the
//    rescoring of a refined layer leaves its candidates' scores by position).
//  - k_cp_merge_compact / k_cp_merge_hist: the gathered pairs of all ranks as
//    one candidate list per row, for the exact selection (the top-k of a
//    union is the top-k of the union of the parts' top-k).
//  - k_cp_combine: split softmax across ranks (each rank's attention kernel
//    leaves its merged partial (acc, m, l)),
//    o = sum_r e^(m_r - M) acc_r / sum_r e^(m_r - M) l_r.
#include <cuda_bf16.h>

#include "cp_internal.cuh"

namespace prism {

constexpr int kCpThreads = 256;
constexpr int kCpSplit = 8;          // CTAs per row of k_cp_prepare

// Grid (rows, kCpSplit): the shard lengths, and the selection's entries
// strided over the row's CTAs.
__global__ void __launch_bounds__(kCpThreads)
k_cp_prepare(CpPrepArgs a) {
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
    for (int t = part * kCpThreads + tid; t < a.src_kappa; t += kCpSplit * kCpThreads) {
        const int p = __ldg(src + t);
        out[t] = (p >= a.lo && p < a.lo + n_loc) ? p - a.lo : -1;
    }
}

cudaError_t launch_cp_prepare(const CpPrepArgs &a, cudaStream_t s) {
    return launch_kernel(k_cp_prepare, dim3(a.B * a.Hkv, kCpSplit), dim3(kCpThreads), 0, s, a);
}

// Grid (ceil(n / kCpThreads), rows): one entry a thread.
__global__ void __launch_bounds__(kCpThreads)
k_cp_pack(CpPackArgs a) {
    const int row = blockIdx.y;
    const int t = blockIdx.x * kCpThreads + threadIdx.x;
    pdl_wait();
    if (t >= a.n) return;
    const int i = __ldcg(a.sel + (size_t)row * a.n + t);
    const bool ok = i >= 0 && i < a.sstride;
    a.pos_out[(size_t)row * a.n + t] = ok ? a.lo + i : -1;
    a.score_out[(size_t)row * a.n + t] = ok ? __ldcg(a.S + (size_t)row * a.sstride + i) : -INFINITY;
}

cudaError_t launch_cp_pack(const CpPackArgs &a, cudaStream_t s) {
    return launch_kernel(k_cp_pack, dim3((a.n + kCpThreads - 1) / kCpThreads, a.rows), dim3(kCpThreads),
                         0, s, a);
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
