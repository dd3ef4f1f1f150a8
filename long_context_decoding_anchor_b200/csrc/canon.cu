// canon.cu -- canonical form of a source selection, for refined layers.
//
// The proposal of a refined layer is every position within r of a previously
// selected index ("Prism Attention", section 3 and Eq. (5), in +-r positional
// form).  Its kernels enumerate that set as disjoint owned ranges, which needs
// the source selection in canonical form: distinct positions in ascending
// order, then -1 padding.  The selections this library produces already are;
// a caller's selection may come in any order, with duplicates.  One CTA per
// (batch, KV head) marks the selected positions in a shared-memory bitmap
// (duplicates vanish there) and a block-wide popcount scan writes them back in
// ascending order, followed (when asked) by the enumeration offsets of the
// proposal around them.
#include "prism_internal.cuh"

namespace prism {

constexpr int kCanonThreads = 1024;

__global__ void __launch_bounds__(kCanonThreads)
k_canonicalize(CanonArgs a) {
    extern __shared__ uint32_t bitmap[];
    __shared__ int scratch[40];
    const int row = blockIdx.x;
    const int b = row / a.Hkv;
    const int tid = threadIdx.x;
    const int L = load_len(a.len, b, a.Lmax, a.st, kWhereCanon);
    const int words = (L + 31) >> 5;
    pdl_wait();

    for (int w = tid; w < words; w += blockDim.x) bitmap[w] = 0u;
    __syncthreads();
    const int32_t *idx = a.idx + (size_t)row * a.kappa;
    for (int t = tid; t < a.kappa; t += blockDim.x) {
        const int i = __ldg(idx + t);
        if (i < 0) continue;
        if (i >= L) {
            report(a.st, kDevErrBadIndex, kWhereCanon, (uint32_t)i);
            continue;
        }
        atomicOr(&bitmap[i >> 5], 1u << (i & 31));
    }
    __syncthreads();

    const int seg = (words + blockDim.x - 1) / blockDim.x;
    const int w_begin = min(words, tid * seg), w_end = min(words, w_begin + seg);
    int cnt = 0;
    for (int w = w_begin; w < w_end; ++w) cnt += __popc(bitmap[w]);
    int total;
    int off = block_exclusive_scan(cnt, scratch, &total);
    int32_t *out = a.out + (size_t)row * a.kappa;
    for (int w = w_begin; w < w_end; ++w) {
        uint32_t bits = bitmap[w];
        while (bits) {
            const int bpos = __ffs(bits) - 1;
            bits &= bits - 1;
            if (off < a.kappa) out[off] = (w << 5) + bpos;
            ++off;
        }
    }
    for (int e = total + tid; e < a.kappa; e += blockDim.x) out[e] = -1;
    if (a.out_off) {
        __syncthreads();
        proposal_offsets(out, a.kappa, a.radius, L, a.out_off + (size_t)row * (a.kappa + 1),
                         scratch, a.st);
    }
}

cudaError_t launch_canonicalize(const CanonArgs &a, cudaStream_t s) {
    const int smem = ((a.Lmax + 31) / 32) * 4;
    cudaError_t e = cudaFuncSetAttribute(k_canonicalize,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(k_canonicalize, dim3(a.B * a.Hkv), dim3(kCanonThreads), smem, s, a);
}

}  // namespace prism
