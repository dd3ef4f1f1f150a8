// cp_internal.cuh -- launch interfaces of the context-parallel helper kernels
// (cp.cu): the pieces around the single-GPU kernels that let one rank work
// on its shard of the positions [lo, lo + cap) of every sequence, and merge
// the ranks' results (exact distributed top-k, split softmax).
#pragma once

#include "prism_internal.cuh"

namespace prism {

enum : int { kCpPrepLen = 0, kCpPrepSelection = 1 };

struct CpPrepArgs {
    int what;                  // kCpPrep*
    const int32_t *len;        // GLOBAL lengths [B]
    int B, Hkv, Lmax;          // Lmax: global capacity
    int lo, cap;               // the shard
    int32_t *llen;             // [B] shard lengths, clamp(len - lo, 0, cap)
    // kCpPrepSelection: src is a global selection of src_kappa entries; out
    // receives it in local positions, -1 where outside the shard.
    const int32_t *src;
    int src_kappa;
    int32_t *out;
    int out_kappa;
    DevStatus *st;
};
cudaError_t launch_cp_prepare(const CpPrepArgs &a, cudaStream_t s);

// (global position, score) of each entry of a local selection; S holds the
// scores by local position (row stride sstride).
struct CpPackArgs {
    const int32_t *sel;        // [rows][n] local positions, ascending, -1 padded
    int rows, n, lo;
    const float *S;
    int sstride;
    int32_t *pos_out;          // [rows][n]
    float *score_out;          // [rows][n]
};
cudaError_t launch_cp_pack(const CpPackArgs &a, cudaStream_t s);

// Gathered per-shard lists -> one ascending candidate list per row (scores S,
// positions cpos, row stride cstride), its count at
// count_out[row * (R * n + 1) + R * n], and its first-digit histogram.
struct CpMergeArgs {
    const int32_t *pos;        // [R][rows][n]
    const float *score;
    int R, rows, n, B, Hkv, Lmax;
    const int32_t *len;
    float *S;
    int32_t *cpos;
    int cstride;
    int32_t *count_out;
    uint32_t *hist;            // [rows][kHistBins]
    DevStatus *st;
};
cudaError_t launch_cp_merge_prepare(const CpMergeArgs &a, cudaStream_t s);

// Split-K partials of the attention kernel -> one (acc[d], m, l) per query head.
struct CpCombineArgs {
    const float *part;         // [R][heads][d + 2]
    int R, heads, d;
    void *out;                 // bf16 [heads][d]
};
cudaError_t launch_cp_combine(const CpCombineArgs &a, cudaStream_t s);

}  // namespace prism
