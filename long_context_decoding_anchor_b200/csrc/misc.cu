// misc.cu -- small utility kernels: the diagnostic export of a refined layer's
// proposal set, and the bounded-wait test hook.
#include "prism_internal.cuh"

namespace prism {

// Diagnostic copy of a refined layer's candidates (ascending positions and
// their scores) into caller buffers of capacity cand_cap per row: the
// proposal of the canonical source enumerated by its owned ranges (one
// contiguous run of entries a thread, a block scan), the scores read by
// position.  One block per row.
__global__ void __launch_bounds__(256)
k_export_candidates(const int32_t *src, int E, int radius, const int32_t *len, int Hkv, int Lmax,
                    const float *Spos, int32_t *cand_pos, float *cand_score, int32_t *cand_count,
                    int cand_cap, DevStatus *st) {
    __shared__ int scratch[40];
    pdl_wait();
    const int row = blockIdx.x, tid = threadIdx.x;
    const int L = load_len(len, row / Hkv, Lmax, st, kWhereCanon);
    const int32_t *sr = src + (size_t)row * E;
    const float *sp = Spos + (size_t)row * Lmax;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int j0 = min(E, tid * per), j1 = min(E, j0 + per);
    int cnt = 0;
    for (int j = j0; j < j1; ++j) {
        int lo;
        cnt += owned_range(sr, j, radius, L, &lo, nullptr, 0);
    }
    int total;
    int o = block_exclusive_scan(cnt, scratch, &total);
    if (tid == 0) cand_count[row] = total;
    for (int j = j0; j < j1 && o < cand_cap; ++j) {
        int lo = 0;
        const int c = owned_range(sr, j, radius, L, &lo, nullptr, 0);
        for (int t = 0; t < c && o < cand_cap; ++t, ++o) {
            cand_pos[(size_t)row * cand_cap + o] = lo + t;
            cand_score[(size_t)row * cand_cap + o] = sp[lo + t];
        }
    }
}

cudaError_t launch_export_candidates(const int32_t *src, int E, int radius, const int32_t *len,
                                     int B, int Hkv, int Lmax, const float *Spos,
                                     int32_t *cand_pos, float *cand_score, int32_t *cand_count,
                                     int cand_cap, DevStatus *st, cudaStream_t s) {
    return launch_kernel(k_export_candidates, dim3(B * Hkv), dim3(256), 0, s, src, E, radius, len,
                         Hkv, Lmax, Spos, cand_pos, cand_score, cand_count, cand_cap, st);
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
