// misc.cu -- small utility kernels: the diagnostic export of a refined layer's
// proposal set, and the bounded-wait test hook.
#include "prism_internal.cuh"

namespace prism {

__global__ void k_export_candidates(const float *S, const int32_t *cpos, const RowCtl *ctl,
                                    int Lmax, int32_t *cand_pos, float *cand_score,
                                    int32_t *cand_count, int cand_cap) {
    const int row = blockIdx.y;
    const int n = ctl[row].n_prop;
    if (blockIdx.x == 0 && threadIdx.x == 0) cand_count[row] = n;
    const int lim = min(n, cand_cap);
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < lim; e += gridDim.x * blockDim.x) {
        cand_pos[(size_t)row * cand_cap + e] = cpos[(size_t)row * Lmax + e];
        cand_score[(size_t)row * cand_cap + e] = S[(size_t)row * Lmax + e];
    }
}

cudaError_t launch_export_candidates(const float *S, const int32_t *cpos, const RowCtl *ctl,
                                     int rows, int Lmax, int32_t *cand_pos, float *cand_score,
                                     int32_t *cand_count, int cand_cap, cudaStream_t s) {
    const int blocks = max(1, min(64, (cand_cap + 255) / 256));
    k_export_candidates<<<dim3(blocks, rows), 256, 0, s>>>(S, cpos, ctl, Lmax, cand_pos,
                                                           cand_score, cand_count, cand_cap);
    count_launches(1);
    return cudaGetLastError();
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
    k_debug_wait<<<1, 32, 0, s>>>(st, limit_ns);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace prism
