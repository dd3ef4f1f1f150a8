// expand.cu -- positional proposal of a refined layer.
//
// P = { p : |p - i| <= r for some selected i of the source layer, 0 <= p < len }
// is the expanded candidate region that a refined layer rescores ("Prism
// Attention", section 3 and section 4.1, Eq. (5)), in its +-r positional form.
// One CTA per (batch, KV head) marks the windows in a shared-memory bitmap
// (duplicates and overlaps vanish there), then a block-wide popcount scan
// writes the set positions in ascending order.
#include "prism_internal.cuh"

namespace prism {

constexpr int kExpandThreads = 1024;

__global__ void __launch_bounds__(kExpandThreads)
k_expand(ExpandArgs a) {
    extern __shared__ uint32_t bitmap[];
    __shared__ int scratch[40];
    const int row = blockIdx.x;
    const int b = row / a.Hkv;
    const int tid = threadIdx.x;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereExpand);
    const int words = (L + 31) >> 5;

    for (int w = tid; w < words; w += blockDim.x) bitmap[w] = 0u;
    __syncthreads();

    const int32_t *prev = a.idx_prev + (size_t)row * a.kappa;
    for (int t = tid; t < a.kappa; t += blockDim.x) {
        const int i = __ldg(prev + t);
        if (i < 0) continue;
        if (i >= L) {
            report(a.st, kDevErrBadIndex, kWhereExpand, (uint32_t)i);
            continue;
        }
        const long long lo = max(0LL, (long long)i - a.radius);
        const long long hi = min((long long)L - 1, (long long)i + a.radius);
        const int w0 = (int)(lo >> 5), w1 = (int)(hi >> 5);
        const uint32_t m0 = 0xffffffffu << (lo & 31);
        const uint32_t m1 = 0xffffffffu >> (31 - (hi & 31));
        if (w0 == w1) {
            atomicOr(&bitmap[w0], m0 & m1);
        } else {
            atomicOr(&bitmap[w0], m0);
            for (int w = w0 + 1; w < w1; ++w) atomicOr(&bitmap[w], 0xffffffffu);
            atomicOr(&bitmap[w1], m1);
        }
    }
    __syncthreads();

    // Ascending enumeration: thread t owns a contiguous segment of words.
    const int seg = (words + blockDim.x - 1) / blockDim.x;
    const int w_begin = min(words, tid * seg), w_end = min(words, w_begin + seg);
    int cnt = 0;
    for (int w = w_begin; w < w_end; ++w) cnt += __popc(bitmap[w]);
    int total;
    int off = block_exclusive_scan(cnt, scratch, &total);
    int32_t *out = a.cpos + (size_t)row * a.Lmax;
    for (int w = w_begin; w < w_end; ++w) {
        uint32_t bits = bitmap[w];
        while (bits) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1;
            out[off++] = (w << 5) + bpos;
        }
    }
    if (tid == 0) a.ctl[row].n_prop = total;
}

cudaError_t launch_expand(const ExpandArgs &a, cudaStream_t s) {
    const int smem = ((a.Lmax + 31) / 32) * 4;
    cudaError_t e = cudaFuncSetAttribute(k_expand, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_expand<<<a.B * a.Hkv, kExpandThreads, smem, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace prism
