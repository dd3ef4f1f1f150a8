// misc.cu -- small utility kernels: the diagnostic export of a refined layer's
// proposal set, and the bounded-wait test hook.
#include "prism_internal.cuh"

namespace prism {

// The proposal of a refined layer in ascending order, with its scores: the
// owned ranges of the canonical source selection, enumerated by one CTA per
// row.
__global__ void __launch_bounds__(512)
k_export_candidates(const float *S, const int32_t *src, const int32_t *len, int Hkv, int Lmax,
                    int kappa, int radius, int32_t *cand_pos, float *cand_score,
                    int32_t *cand_count, int cand_cap, DevStatus *st) {
    __shared__ int scratch[40];
    const int row = blockIdx.x, tid = threadIdx.x;
    const int L = load_len(len, row / Hkv, Lmax, st, kWhereCanon);
    const int32_t *s = src + (size_t)row * kappa;
    int running = 0;
    for (int jb = 0; jb < kappa; jb += blockDim.x) {
        int lo = 0, cnt = 0;
        if (jb + tid < kappa) cnt = owned_range(s, jb + tid, radius, L, &lo, st, kWhereCanon);
        int tot;
        const int ex = block_exclusive_scan(cnt, scratch, &tot);
        for (int i = 0; i < cnt; ++i) {
            const int o = running + ex + i;
            if (o < cand_cap) {
                cand_pos[(size_t)row * cand_cap + o] = lo + i;
                cand_score[(size_t)row * cand_cap + o] = S[(size_t)row * Lmax + lo + i];
            }
        }
        running += tot;
    }
    if (tid == 0) cand_count[row] = running;
}

cudaError_t launch_export_candidates(const float *S, const int32_t *src, const RowCtl *,
                                     const int32_t *len, int B, int Hkv, int Lmax, int kappa,
                                     int radius, int32_t *cand_pos, float *cand_score,
                                     int32_t *cand_count, int cand_cap, DevStatus *st,
                                     cudaStream_t s) {
    k_export_candidates<<<B * Hkv, 512, 0, s>>>(S, src, len, Hkv, Lmax, kappa, radius, cand_pos,
                                                cand_score, cand_count, cand_cap, st);
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
