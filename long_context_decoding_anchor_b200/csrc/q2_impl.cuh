// q2_impl.cuh -- the 2-bit proposal keys of "Prism Attention" (section 4.2,
// Eq. (7)-(9)): the row format, and the group-maximum scores of 16 key rows
// by one warp on the tensor cores.
//
// Row format (one key row of d elements, kQ2RowBytes(d) = d / 2 bytes):
//   bytes [0, d/4)       the 2-bit codes.  A 16-element k step kk of the row
//                        holds, for t = 0..3, the codes of elements 16kk + 2t,
//                        16kk + 2t + 1, 16kk + 2t + 8 and 16kk + 2t + 9 (bits
//                        0-1, 2-3, 4-5, 6-7) in byte t * (d/16) + kk: lane t of
//                        an mma.sync quad finds its codes of every k step in
//                        d/16 consecutive bytes.
//   bytes [d/4, d/2)     per group m of kQ2Group elements, alpha_m then beta_m
//                        (fp32): the element with code c stands for
//                        alpha_m * c + beta_m (Eq. (8) read back).
//
// Scores: a warp's 16 rows against the group's query heads by mma.sync
// m16n8k16 (bf16 in, fp32 accumulate), one accumulator per group.  The codes
// enter the A fragments as the bf16 numbers 128 + c (exact); the epilogue
// takes off 128 * sum(q over the group) again:
//   <q_j, khat_i> = sum_m alpha_m (acc_m - 128 S_jm) + beta_m S_jm,
//   S_jm = sum over group m of q_j.
#pragma once

#include "prism_internal.cuh"

namespace prism {

constexpr int kQ2Group = 32;
__host__ __device__ constexpr int q2_row_bytes(int d) { return d / 2; }

// Two bf16 (128 + c_lo, 128 + c_hi) from two 2-bit codes.
__device__ __forceinline__ uint32_t q2_pair(uint32_t two_codes) {
    return 0x43004300u | (two_codes & 3u) | ((two_codes & 0xcu) << 14);
}

// The quad lane's A fragment registers of k step kk for rows g and g + 8,
// from their code bytes (byte kk of the lane's d/16 consecutive bytes).
__device__ __forceinline__ void q2_afrag(uint32_t byte_g, uint32_t byte_g8, uint32_t &a0,
                                         uint32_t &a1, uint32_t &a2, uint32_t &a3) {
    a0 = q2_pair(byte_g);            // row g,     k 2t, 2t+1
    a1 = q2_pair(byte_g8);           // row g + 8, k 2t, 2t+1
    a2 = q2_pair(byte_g >> 4);       // row g,     k 2t+8, 2t+9
    a3 = q2_pair(byte_g8 >> 4);      // row g + 8, k 2t+8, 2t+9
}

__device__ __forceinline__ void mma16816_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The group's queries as the warp needs them (one KV head of one sequence).
// qf: B fragments (column n of n-tile u is head (8u + n) % G; k pairs
// 2*(lane%4) and +8 of each k step).  S: sum over each group m of the
// elements of the heads this lane's accumulator columns hold (heads
// (8u + 2*(lane%4)) % G and (8u + 2*(lane%4) + 1) % G).
template <int D, int NT>
struct Q2Query {
    uint32_t qf[NT][D / 16][2];
    float S[NT][D / kQ2Group][2];
};

// NT n-tiles of 8 heads: 1 for G <= 8, 2 for G = 16.
template <int D, int NT>
__device__ __forceinline__ void q2_load_query(Q2Query<D, NT> &Q, const uint16_t *qg, int G, int lane) {
#pragma unroll
    for (int u = 0; u < NT; ++u) {
        const uint16_t *qh = qg + (size_t)((8 * u + (lane >> 2)) % G) * D + 2 * (lane & 3);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            Q.qf[u][kk][0] = *reinterpret_cast<const uint32_t *>(qh + 16 * kk);
            Q.qf[u][kk][1] = *reinterpret_cast<const uint32_t *>(qh + 16 * kk + 8);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint16_t *qc = qg + (size_t)((8 * u + 2 * (lane & 3) + c) % G) * D;
#pragma unroll
            for (int m = 0; m < D / kQ2Group; ++m) {
                float s = 0.f;
                for (int e = 0; e < kQ2Group; ++e)
                    s += __uint_as_float((uint32_t)qc[m * kQ2Group + e] << 16);
                Q.S[u][m][c] = s;
            }
        }
    }
}

// Group maxima (Eq. (9), unscaled) of NS blocks of 16 rows (rows at stride
// q2_row_bytes(D), block i starting at rows16 + i * block_stride bytes, in
// shared memory), computed side by side so that their latency chains
// overlap: out[i].x for row lane/4 of block i, out[i].y for row lane/4 + 8,
// in every lane of the quad.
template <int D, int NT, int NS>
__device__ __forceinline__ void q2_group_max_rows(const uint8_t *rows16, int block_stride,
                                                  const Q2Query<D, NT> &Q, int lane,
                                                  float2 (&out)[NS]) {
    constexpr int RB = q2_row_bytes(D);
    constexpr int KS = D / 16;
    constexpr int KW = KS / 4 > 0 ? KS / 4 : 1;
    constexpr int M = D / kQ2Group;
    const int g = lane >> 2, t = lane & 3;
    uint32_t w0[NS][KW], w1[NS][KW];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const uint8_t *r0 = rows16 + i * block_stride + g * RB, *r1 = r0 + 8 * RB;
#pragma unroll
        for (int j = 0; j < KW; ++j) {
            w0[i][j] = *reinterpret_cast<const uint32_t *>(r0 + t * KS + 4 * j);
            w1[i][j] = *reinterpret_cast<const uint32_t *>(r1 + t * KS + 4 * j);
        }
    }
    float acc[NS][NT][M][4];
#pragma unroll
    for (int i = 0; i < NS; ++i)
#pragma unroll
        for (int u = 0; u < NT; ++u)
#pragma unroll
            for (int m = 0; m < M; ++m)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][u][m][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        const int m = kk / (kQ2Group / 16);
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const uint32_t b0 = (w0[i][kk >> 2] >> (8 * (kk & 3))) & 0xffu;
            const uint32_t b1 = (w1[i][kk >> 2] >> (8 * (kk & 3))) & 0xffu;
            uint32_t a0, a1, a2, a3;
            q2_afrag(b0, b1, a0, a1, a2, a3);
#pragma unroll
            for (int u = 0; u < NT; ++u)
                mma16816_bf16(acc[i][u][m], a0, a1, a2, a3, Q.qf[u][kk][0], Q.qf[u][kk][1]);
        }
    }
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const uint8_t *r0 = rows16 + i * block_stride + g * RB, *r1 = r0 + 8 * RB;
        float lo = -INFINITY, hi = -INFINITY;
#pragma unroll
        for (int u = 0; u < NT; ++u) {
            float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;  // (row g | g+8) x (column 2t | 2t+1)
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const float2 p0 = *reinterpret_cast<const float2 *>(r0 + D / 4 + 8 * m);   // alpha, beta
                const float2 p1 = *reinterpret_cast<const float2 *>(r1 + D / 4 + 8 * m);
                const float Sa = Q.S[u][m][0], Sb = Q.S[u][m][1];
                s00 += p0.x * (acc[i][u][m][0] - 128.f * Sa) + p0.y * Sa;
                s01 += p0.x * (acc[i][u][m][1] - 128.f * Sb) + p0.y * Sb;
                s10 += p1.x * (acc[i][u][m][2] - 128.f * Sa) + p1.y * Sa;
                s11 += p1.x * (acc[i][u][m][3] - 128.f * Sb) + p1.y * Sb;
            }
            lo = fmaxf(lo, fmaxf(s00, s01));
            hi = fmaxf(hi, fmaxf(s10, s11));
        }
        lo = fmaxf(lo, __shfl_xor_sync(0xffffffffu, lo, 1));
        lo = fmaxf(lo, __shfl_xor_sync(0xffffffffu, lo, 2));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 1));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 2));
        out[i] = make_float2(lo, hi);
    }
}

template <int D, int NT>
__device__ __forceinline__ float2 q2_group_max_16rows(const uint8_t *rows16, const Q2Query<D, NT> &Q,
                                                      int lane) {
    float2 o[1];
    q2_group_max_rows<D, NT, 1>(rows16, 0, Q, lane, o);
    return o[0];
}

}  // namespace prism
