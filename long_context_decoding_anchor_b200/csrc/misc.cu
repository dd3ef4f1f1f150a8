// misc.cu -- small utility kernels: the diagnostic export of a refined layer's
// proposal set, and the bounded-wait test hook.
#include "prism_internal.cuh"

namespace prism {

// Diagnostic copy of a refined layer's candidates (ascending positions and
// their scores) into caller buffers of capacity cand_cap per row.
__global__ void __launch_bounds__(256)
k_export_candidates(const float *cscore, const int32_t *cpos, const int32_t *src_off, int Lmax,
                    int kappa, int32_t *cand_pos, float *cand_score, int32_t *cand_count,
                    int cand_cap) {
    pdl_wait();
    const int row = blockIdx.y;
    const int n = min(src_off[(size_t)row * (kappa + 1) + kappa], Lmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) cand_count[row] = n;
    const int lim = min(n, cand_cap);
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < lim; e += gridDim.x * blockDim.x) {
        cand_pos[(size_t)row * cand_cap + e] = cpos[(size_t)row * Lmax + e];
        cand_score[(size_t)row * cand_cap + e] = cscore[(size_t)row * Lmax + e];
    }
}

cudaError_t launch_export_candidates(const float *cscore, const int32_t *cpos,
                                     const int32_t *src_off, int rows, int Lmax, int kappa,
                                     int32_t *cand_pos, float *cand_score, int32_t *cand_count,
                                     int cand_cap, cudaStream_t s) {
    const int blocks = max(1, min(64, (cand_cap + 255) / 256));
    return launch_kernel(k_export_candidates, dim3(blocks, rows), dim3(256), 0, s, cscore, cpos,
                         src_off, Lmax, kappa, cand_pos, cand_score, cand_count, cand_cap);
}

// Waits on an mbarrier that nothing will ever complete, for at most limit_ns,
// then records a timeout.  Exercises the same bounded-wait path as the
// pipelined kernels, without any risk of a hang.
__global__ void k_debug_wait(DevStatus *st, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait(&bar, 0u, limit_ns)) report(st, kDevErrTimeout, kWhereDebugWait, 0u);
        // Complete the phase so that nothing is left pending at exit.
        mbar_arrive(&bar);
    }
}

cudaError_t launch_debug_wait(DevStatus *st, uint64_t limit_ns, cudaStream_t s) {
    return launch_kernel(k_debug_wait, dim3(1), dim3(32), 0, s, st, limit_ns);
}

}  // namespace prism
