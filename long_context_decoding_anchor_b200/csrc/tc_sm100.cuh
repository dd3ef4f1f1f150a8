// tc_sm100.cuh -- the sm_100a tensor-core (tcgen05) and tensor-TMA primitives
// used by the group-maximum scoring kernel: tensor memory allocation, the
// shared-memory matrix and instruction descriptors of tcgen05.mma (kind::f16,
// bf16 operands, fp32 accumulator), commits to mbarriers, tensor-memory loads,
// and the 2-D tiled TMA load with 128-byte swizzle.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "prism_internal.cuh"

namespace prism {

// ---- tensor memory --------------------------------------------------------
// Allocation of `ncols` columns (a power of two >= 32) by one whole warp; the
// base address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Generic-proxy writes to shared memory become visible to the async proxy
// (TMA, tensor cores) of this CTA.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- tcgen05.mma descriptors ----------------------------------------------
// Shared-memory matrix descriptor of a K-major operand stored in the
// 128-byte-swizzle canonical layout: rows of 128 bytes (64 bf16 of K), the
// 16-byte chunk c of row r stored at chunk c ^ (r % 8), groups of 8 rows 1024
// bytes apart.  Fields: start address >> 4 (bits 0-13), leading byte offset
// >> 4 (16-29; unused by this layout, 1 by convention), stride byte offset
// >> 4 (32-45) = 1024 >> 4, descriptor version 1 (46-47), base offset 0
// (49-51; the atoms are 1024-byte aligned), layout 2 = 128-byte swizzle
// (61-63).  A K step of 16 elements inside the 64-element atom advances the
// start address by 32 bytes.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3fffu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B, fp32
// accumulator, both operands K-major, no negation: accumulator format F32
// (bits 4-5 = 1), A format BF16 (7-9 = 1), B format BF16 (10-12 = 1), N >> 3
// (17-22), M >> 4 (24-28).
template <int M, int N>
__device__ __forceinline__ constexpr uint32_t idesc_bf16_f32() {
    static_assert(M == 64 || M == 128, "M of a single-CTA MMA");
    static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N of an M=128 MMA");
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// The mbarrier receives one arrival once every tcgen05 operation issued so far
// by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                     "r"(smem_addr(bar))
                 : "memory");
}

// 32 lanes x 16 columns of 32 bits: thread i of the warp receives lane
// (base lane + i), columns [col, col + 16).  The warp may only address the
// 32-lane quarter (warp id % 4) of tensor memory.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- 2-D tiled TMA load -----------------------------------------------------
// Box at element coordinates (x, y) of the tensor map into shared memory,
// completing on `bar`.  x * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

}  // namespace prism
