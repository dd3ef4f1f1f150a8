// tiles.cuh -- the tile order of a full-cache scan: every (batch, KV head)
// row's context split into tiles of TILE key rows, rows in (b, h) order, and
// a persistent CTA's walk over its contiguous share of that order.
#pragma once

#include "prism_internal.cuh"

namespace prism {

// Position of tile `t` of the global tile order (row-major over (b, h), then
// tile j) given tiles_b = ceil(len[b] / TILE).  Found by a block-wide scan over
// the batch; every thread of the block gets the result.
struct TileCursor {
    int b, h, j, tiles_b;
};

template <int TILE>
__device__ void locate_tile(const int32_t *len, int B, int Hkv, int Lmax, long long t,
                            TileCursor *cur, long long *total, int *scratch, DevStatus *st) {
    long long base = 0;  // tiles of all (b, h) before the current batch chunk
    __shared__ long long s_found_base;
    __shared__ int s_found_b;
    __syncthreads();   // earlier readers of s_found_b are done
    if (threadIdx.x == 0) s_found_b = -1;
    __syncthreads();
    for (int b0 = 0; b0 < B; b0 += blockDim.x) {
        const int b = b0 + threadIdx.x;
        int tb = 0;
        if (b < B) {
            int L = load_len(len, b, Lmax, st, kWhereScore);
            tb = (L + TILE - 1) / TILE;
        }
        int tot;
        int ex = block_exclusive_scan(tb, scratch, &tot);
        long long my0 = base + (long long)ex * Hkv;
        long long my1 = my0 + (long long)tb * Hkv;
        if (b < B && tb > 0 && t >= my0 && t < my1) {
            s_found_b = b;
            s_found_base = my0;
        }
        base += (long long)tot * Hkv;
    }
    __syncthreads();
    *total = base;
    if (s_found_b >= 0) {
        const int b = s_found_b;
        int L = __ldg(len + b);
        L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
        const int tb = (L + TILE - 1) / TILE;
        const long long rem = t - s_found_base;
        cur->b = b;
        cur->h = (int)(rem / tb);
        cur->j = (int)(rem % tb);
        cur->tiles_b = tb;
    } else {
        cur->b = B;
        cur->h = 0;
        cur->j = 0;
        cur->tiles_b = 0;
    }
}

// Advance to the next tile (skipping empty sequences).
template <int TILE>
__device__ __forceinline__ void next_tile(TileCursor &c, const int32_t *len, int B, int Hkv,
                                          int Lmax) {
    if (++c.j < c.tiles_b) return;
    c.j = 0;
    if (++c.h < Hkv) return;
    c.h = 0;
    for (++c.b; c.b < B; ++c.b) {
        int L = __ldg(len + c.b);
        L = L < 0 ? 0 : (L > Lmax ? Lmax : L);
        c.tiles_b = (L + TILE - 1) / TILE;
        if (c.tiles_b > 0) return;
    }
}

}  // namespace prism
