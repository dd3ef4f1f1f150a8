// prism_internal.cuh -- device helpers and launch interfaces shared by the
// kernels of the Prism Attention decode hot path (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace prism {

// First-level radix digit of a score key (the top 11 bits).
constexpr int kHistBits = 11;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kMaxLen = 1 << 20;

// Device status word (first bytes of the workspace).
struct DevStatus {
    uint32_t code;    // 0 = ok, else one of the kDevErr* values
    uint32_t where;   // which kernel reported
    uint32_t value;   // offending value (a length, an index, a stage)
    uint32_t pad;
};
enum : uint32_t {
    kDevErrNone = 0,
    kDevErrTimeout = 1,
    kDevErrBadLen = 2,
    kDevErrBadIndex = 3,
    kDevErrInternal = 4,
};
enum : uint32_t {
    kWhereScore = 1,
    kWhereRescore = 2,
    kWhereCanon = 3,
    kWhereCollect = 4,
    kWhereFinalize = 5,
    kWhereAttn = 6,
    kWhereDebugWait = 7,
};

// Per (batch, KV head) row counter of the attention kernel's split-K merge;
// zeroed at the start of every public call that uses it and left zeroed.
struct RowCtl {
    uint32_t done_attn;    // attention CTAs of this row that have finished
    uint32_t pad[7];
};

__device__ __forceinline__ void report(DevStatus *st, uint32_t code, uint32_t where,
                                       uint32_t value) {
    if (atomicCAS(&st->code, 0u, code) == 0u) {
        st->where = where;
        st->value = value;
    }
}

// Clamped context length of batch entry b (reports values outside [0, Lmax]).
__device__ __forceinline__ int load_len(const int32_t *len, int b, int Lmax, DevStatus *st,
                                        uint32_t where) {
    int L = __ldg(len + b);
    if (L < 0 || L > Lmax) {
        report(st, kDevErrBadLen, where, (uint32_t)L);
        L = L < 0 ? 0 : Lmax;
    }
    return L;
}

// Order-preserving unsigned key of an fp32 score: a > b  <=>  key(a) > key(b).
// -0.0 is folded onto +0.0 so the two tie.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    u = (u == 0x80000000u) ? 0u : u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// bf16 halves of a 32-bit word, widened exactly to fp32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// <k, q> over 8 bf16 key elements and 8 fp32 query elements: two fp32
// accumulators (even and odd elements), each a chain of round-to-nearest FMAs
// issued in pairs (fma.rn.f32x2), added at the end.  Every kernel that scores
// with it forms bit-identical scores for the same key and query.
__device__ __forceinline__ unsigned long long f32x2_pack(float lo, float hi) {
    return ((unsigned long long)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ unsigned long long fma_f32x2(unsigned long long a, unsigned long long b,
                                                        unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float dot8(const uint4 &kv, const float *q) {
    // word w holds elements 2w (low half) and 2w + 1 (high half); the
    // accumulators start at -0.0, so the first step is exactly a product
    // (signed zeros survive: a key of -0.0 scores -0.0)
    unsigned long long acc = 0x8000000080000000ull;
    acc = fma_f32x2(((unsigned long long)(kv.x & 0xffff0000u) << 32) | (kv.x << 16), f32x2_pack(q[0], q[1]), acc);
    acc = fma_f32x2(((unsigned long long)(kv.y & 0xffff0000u) << 32) | (kv.y << 16), f32x2_pack(q[2], q[3]), acc);
    acc = fma_f32x2(((unsigned long long)(kv.z & 0xffff0000u) << 32) | (kv.z << 16), f32x2_pack(q[4], q[5]), acc);
    acc = fma_f32x2(((unsigned long long)(kv.w & 0xffff0000u) << 32) | (kv.w << 16), f32x2_pack(q[6], q[7]), acc);
    return __uint_as_float((uint32_t)acc) + __uint_as_float((uint32_t)(acc >> 32));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Programmatic dependent launch: wait for the preceding kernel of the stream
// (and the visibility of its writes); let the next kernel start its prologue.
// Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Transposing butterfly reduction.  Each lane of an NL-lane group holds NV
// partial sums (one per item); after the call the lane holds in v[0] the full
// group sum of item `transpose_item<NV, NL>(lane)` (for NV <= NL).  Costs
// NV-1 + log2(NL/NV) shuffles instead of NV*log2(NL).
template <int NV, int NL>
__device__ __forceinline__ void transpose_reduce(float (&v)[NV], int lane) {
    static_assert((NV & (NV - 1)) == 0 && (NL & (NL - 1)) == 0, "powers of two");
    static_assert(NV <= NL, "at most one item per lane after the reduction");
    int cnt = NV;
#pragma unroll
    for (int m = NL / 2; m >= 1; m >>= 1) {
        if (cnt > 1) {
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < NV / 2; ++i) {
                if (i < cnt / 2) {
                    float keep = upper ? v[i + cnt / 2] : v[i];
                    float send = upper ? v[i] : v[i + cnt / 2];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            cnt >>= 1;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
        }
    }
}

// Which item a lane holds after transpose_reduce<NV, NL>.
template <int NV, int NL>
__device__ __forceinline__ int transpose_item(int lane) {
    int item = 0;
    int bit = NV / 2;
#pragma unroll
    for (int m = NL / 2; m >= 1 && bit >= 1; m >>= 1, bit >>= 1)
        if (lane & m) item |= bit;
    return item;
}

// Whether this lane is the one (of NL/NV equal copies) that stores the item.
template <int NV, int NL>
__device__ __forceinline__ bool transpose_writer(int lane) {
    return (lane & (NL / NV - 1)) == 0;
}

// ---- positional proposal: owned ranges ------------------------------------
// A canonical selection lists distinct positions in ascending order, then -1
// padding.  With it, the proposal P = union of [i - r, i + r] clipped to
// [0, L) splits into disjoint consecutive ranges: entry j owns the positions of
// its window that no earlier entry's window covers,
//   lo_j = max(i_j - r, i_{j-1} + r + 1, 0),  hi_j = min(i_j + r, L - 1),
// so P is enumerated in ascending order, without duplicates, entry by entry.
// A malformed entry (>= L, or not above its predecessor) is reported and owns
// nothing; the ranges stay inside [0, L) either way.
__device__ __forceinline__ int owned_range(const int32_t *src, int j, long long r, int L,
                                           int *lo_out, DevStatus *st, uint32_t where) {
    const int i = src[j];
    if (i < 0) return 0;
    const int prev = j > 0 ? src[j - 1] : -1;
    if (i >= L || (prev >= 0 && i <= prev)) {
        if (st) report(st, kDevErrBadIndex, where, (uint32_t)i);
        return 0;
    }
    long long lo = (long long)i - r;
    if (prev >= 0 && (long long)prev + r + 1 > lo) lo = (long long)prev + r + 1;
    if (lo < 0) lo = 0;
    long long hi = (long long)i + r;
    if (hi > L - 1) hi = L - 1;
    if (hi < lo) return 0;
    *lo_out = (int)lo;
    return (int)(hi - lo + 1);
}

// One entry of the source selection as the producer lane sees it: its slots
// [o0, o1) of the enumeration and the first key row `lo` of its owned range.
// The raw loads are issued one batch ahead of their use.
struct EntryRaw {
    int o0, o1, i, prev;
};
struct EntryRun {
    int o0, o1, lo;
};

__device__ __forceinline__ EntryRaw load_entry_raw(const int32_t *src, const int32_t *off,
                                                   int kappa, int jj) {
    EntryRaw w{-1, -1, -1, -1};
    if (jj < kappa) {
        w.o0 = __ldcg(off + jj);
        w.o1 = __ldcg(off + jj + 1);
        w.i = __ldcg(src + jj);
        w.prev = jj > 0 ? __ldcg(src + jj - 1) : -1;
    }
    return w;
}

__device__ __forceinline__ EntryRun make_entry(const EntryRaw &w, int jj, int kappa, int n,
                                               long long r, int L, DevStatus *st) {
    EntryRun e{n, n, 0};
    if (jj >= kappa) return e;
    e.o0 = min(w.o0, n);
    e.o1 = min(w.o1, n);
    long long lo = (long long)w.i - r;
    if (w.prev >= 0 && (long long)w.prev + r + 1 > lo) lo = (long long)w.prev + r + 1;
    if (lo < 0) lo = 0;
    long long hi = (long long)w.i + r;
    if (hi > L - 1) hi = L - 1;
    const int own = (w.i < 0 || hi < lo) ? 0 : (int)(hi - lo + 1);
    if (e.o1 - e.o0 != own && e.o1 > e.o0) {
        report(st, kDevErrInternal, kWhereRescore, (uint32_t)jj);   // offsets disagree
        lo = 0;
    }
    e.lo = (int)lo;
    return e;
}

// ---- mbarrier / bulk-copy (TMA) primitives -------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase of `parity` to complete; false after limit_ns
// (or after an iteration cap, should the timer misbehave).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0; it < (1u << 28); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 31u && global_timer_ns() - t0 > limit_ns) return false;
    }
    return false;
}
// Acquire load at GPU scope (pairs with a fence + atomic arrival elsewhere).
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Barrier of blocks that are resident together (the caller guarantees it):
// thread 0 makes the block's earlier global writes visible, adds one arrival
// to *ctr and waits until *ctr reaches `target`, bounded by limit_ns (then it
// records a timeout and lets the block continue; the results are void).  The
// whole block calls it; *ok (shared) says whether the wait completed.
__device__ __forceinline__ void block_group_barrier(uint32_t *ctr, uint32_t target, uint64_t limit_ns,
                                                    DevStatus *st, uint32_t where, int *ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        // the block's writes (ordered before this thread by the barrier)
        // become visible before the arrival: the fence is cumulative
        __threadfence();
        atomicAdd(ctr, 1u);
        const uint64_t t0 = global_timer_ns();
        int good = 1;
        for (uint32_t it = 0; ld_acquire_gpu(ctr) < target; ++it) {
            if ((it & 15u) == 15u && global_timer_ns() - t0 > limit_ns) {
                report(st, kDevErrTimeout, where, target);
                good = 0;
                break;
            }
        }
        *ok = good;
    }
    __syncthreads();
}

// Evict-first L2 policy for data read exactly once (the streamed key cache).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// 1-D bulk copy global -> shared, completing on `bar` (bytes % 16 == 0, both
// addresses 16-byte aligned).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// ---- cp.async (16-byte) gather primitives ---------------------------------
// src_bytes = 0 zero-fills the destination without reading global memory.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// ---- block-wide exclusive scan (int), blockDim.x a multiple of 32 ---------
// `scratch` holds at least 33 ints.  Returns the exclusive prefix of `x`;
// *total receives the block sum.  Contains __syncthreads().
__device__ __forceinline__ int block_exclusive_scan(int x, int *scratch, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nwarps) scratch[lane] = wi - w;
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    int res = scratch[warp] + incl - x;
    *total = scratch[32];
    __syncthreads();
    return res;
}

// Threshold digit of a histogram: the bin `bsel` such that the number of items
// in bins above it is < need <= that number + hist[bsel].  `hist` is in shared
// memory with `nbins` entries (a multiple of blockDim.x).  Writes bsel and the
// count above it to out[0], out[1].  Contains __syncthreads().
__device__ __forceinline__ void find_threshold_bin(const uint32_t *hist, int nbins, int need,
                                                   int *scratch, int *out) {
    const int per = nbins / blockDim.x;
    // Thread t owns bins [nbins - (t+1)*per, nbins - t*per): thread 0 the top.
    const int hi = nbins - threadIdx.x * per;
    int local = 0;
    for (int i = 1; i <= per; ++i) local += (int)hist[hi - i];
    int total;
    int above = block_exclusive_scan(local, scratch, &total);
    if (above < need && above + local >= need) {
        int acc = above;
        for (int i = 1; i <= per; ++i) {
            int h = (int)hist[hi - i];
            if (acc + h >= need) {
                out[0] = hi - i;
                out[1] = acc;
                break;
            }
            acc += h;
        }
    }
    __syncthreads();
}

// Enumeration of the proposal positions owned by entries [j0, j0 + kPropEntries)
// of a canonical source selection: per-entry range starts in lo_s, exclusive
// offsets in off_s[0..kPropEntries].  Returns the number of positions (all
// threads).  Needs blockDim.x >= kPropEntries.  Contains __syncthreads().
constexpr int kPropEntries = 64;
__device__ __forceinline__ int proposal_slice(const int32_t *src_row, int j0, int kappa,
                                              int radius, int L, int *lo_s, int *off_s,
                                              int *scratch, DevStatus *st, uint32_t where) {
    int cnt = 0, lo = 0;
    const int t = threadIdx.x;
    if (t < kPropEntries && j0 + t < kappa)
        cnt = owned_range(src_row, j0 + t, radius, L, &lo, st, where);
    int total;
    const int ex = block_exclusive_scan(t < kPropEntries ? cnt : 0, scratch, &total);
    if (t < kPropEntries) {
        lo_s[t] = lo;
        off_s[t] = ex;
    }
    if (t == 0) off_s[kPropEntries] = total;
    __syncthreads();
    return total;
}

// Position of enumeration index e of a proposal slice.
__device__ __forceinline__ int slice_position(const int *lo_s, const int *off_s, int e) {
    int a = 0, b = kPropEntries - 1;       // largest t with off_s[t] <= e
    while (a < b) {
        const int m = (a + b + 1) >> 1;
        if (off_s[m] <= e) a = m; else b = m - 1;
    }
    return lo_s[a] + (e - off_s[a]);
}

// Enumeration offsets of the proposal around a canonical selection sel[0..kappa):
// off[j] = number of proposal positions owned by entries before j, off[kappa]
// = |P|.  Whole-CTA cooperative; sel may have been written by this CTA
// (call after a barrier).  Contains __syncthreads().
__device__ __forceinline__ void proposal_offsets(const int32_t *sel, int kappa, int radius, int L,
                                                 int32_t *off, int *scratch, DevStatus *st) {
    const int NT = blockDim.x, tid = threadIdx.x;
    const int per = (kappa + NT - 1) / NT;
    const int j0 = min(kappa, tid * per), j1 = min(kappa, j0 + per);
    int cnt = 0;
    for (int j = j0; j < j1; ++j) {
        int lo;
        cnt += owned_range(sel, j, radius, L, &lo, st, kWhereFinalize);
    }
    int total;
    int run = block_exclusive_scan(cnt, scratch, &total);
    for (int j = j0; j < j1; ++j) {
        off[j] = run;
        int lo;
        run += owned_range(sel, j, radius, L, &lo, nullptr, 0);
    }
    if (tid == 0) off[kappa] = total;
}

// ---- launch interfaces (host side, defined in the .cu files) -------------
// Kernels launched by the calling host thread (see prism_launch_count()).
void count_launches(int n);

// Whether kernels are launched with programmatic dependent launch (on unless
// the environment sets PRISM_NO_PDL=1).
bool use_pdl();

// Launch with the programmatic-stream-serialization attribute, so that the
// kernel may begin while its predecessor in the stream finishes (the kernel
// calls pdl_wait() before it touches the predecessor's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = use_pdl() ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
    count_launches(1);
    return e;
}

struct ScoreArgs {
    const void *q;          // bf16 [B][Hq][d]
    const void *k;          // bf16 [B][Hkv][Lmax][d]
    const int32_t *len;     // [B]
    int B, Hkv, G, d, Lmax;
    float scale;
    float *S;               // anchor: fp32 [rows][Lmax] scores by position
    uint32_t *hist;         // [rows][kHistBins] first-digit histogram (accumulated)
    const int32_t *src;     // refine: canonical source selection [rows][kappa]
    int kappa, radius;      // refine: entries of the source selection, proposal radius
    int agg;                // kAggSum: Eq. (1) group sum; kAggMax: Eq. (9) group maximum
    int q2;                 // nonzero: k (and kz) are 2-bit key caches (Eq. (7)-(8),
                            // rows of d/2 bytes, q2_impl.cuh), scored by Eq. (9)
    // refine: the candidates leave as runs (see RefineParts): run t of a row
    // holds run_cnt[row * nruns + t] items (key << 32 | position), ordered by
    // first radix digit, highest first, at runs + (row * nruns + t) * kRunCap
    uint64_t *runs;
    int32_t *run_cnt;
    int parts, run_k;       // parts per row, runs per part (nruns = parts * run_k)
    float *Spos;            // refine, nullable: every candidate's score by position
    int spos_stride;        //   (row stride)
    // refine on one shard of a context-parallel rank (glen nullable): the
    // source holds global positions, len is the shard's, and the proposal is
    // cut to the shard [shard_lo, shard_lo + len) in local positions; glen
    // (capacity glmax) are the global lengths the windows are clipped to
    const int32_t *glen;
    int glmax, shard_lo;
    // refine, fused selection (Eq. (6) in the same launch; nz == 1, one run a
    // part, every block of the grid resident at once): the blocks of a row
    // meet at two barriers on row_bar[row] (arrivals counted from bar_base),
    // exchange their first-digit ties through their runs and their counts
    // through part_cnt [rows][parts][2], and each writes its selected
    // positions to sel_out [rows][kap_out] at its offset; ties beyond the
    // shared-memory cache go to tie_spill [rows][tie_cap]
    int fused;
    int two_stages;         // group sum: the smaller rescoring CTA (two gather stages)
    uint32_t *row_bar;
    uint32_t bar_base;
    int32_t *part_cnt;
    int32_t *sel_out;
    int kap_out;
    uint64_t *tie_spill;
    int tie_cap;
    // refine: several layers rescoring the same source in one launch (grid z);
    // layer z reads qz[z] / kz[z] (z = 0: q / k) and writes runs, run_cnt and
    // hist shifted by z * zruns, z * zcnt, z * zhist
    int nz;
    const void *qz[8];
    const void *kz[8];
    size_t zruns, zcnt, zhist;
    DevStatus *st;
    uint64_t wait_ns;
};
// Work split of a refined layer's rescoring.  Part p of a row takes the
// source entries [p*E/P, (p+1)*E/P) -- at most kMaxPartEntries -- and the
// proposal positions they own, at most run_k * kRunCap of them; each run of
// kRunCap candidates is sorted by first digit for the selection.
constexpr int kRunCap = 2048;
constexpr int kMaxPartEntries = 512;
constexpr int kTargetCtas = 148;   // rescoring blocks aimed at per launch (B200 SMs)
struct RefineParts {
    int parts, run_k;
};
inline RefineParts refine_parts(int E, int radius, int Lmax, int rows, int nz) {
    const long long own = (long long)2 * radius + 1 < Lmax ? 2LL * radius + 1 : (long long)Lmax;
    const long long per_run = own <= kRunCap ? kRunCap / own : 1;        // entries a run holds
    long long per = per_run < kMaxPartEntries ? per_run : kMaxPartEntries;
    long long P = (E + per - 1) / per;
    const long long want = kTargetCtas / ((long long)rows * (nz > 0 ? nz : 1));
    if (P < want) P = want < E ? want : E;
    if (P < 1) P = 1;
    const long long ent = (E + P - 1) / P;                                // entries of a part
    long long slots = ent * own;
    if (slots > Lmax) slots = Lmax;
    RefineParts r;
    r.parts = (int)P;
    r.run_k = (int)((slots + kRunCap - 1) / kRunCap);
    if (r.run_k < 1) r.run_k = 1;
    return r;
}
enum : int { kAggSum = 0, kAggMax = 1 };
constexpr int kMaxZ = 8;           // refined layers batched into one launch

cudaError_t launch_anchor_score(const ScoreArgs &a, int num_sms, cudaStream_t s);
// The group-maximum form of the full-cache scan (tensor cores; score_max.cu).
cudaError_t launch_anchor_score_max(const ScoreArgs &a, int num_sms, cudaStream_t s);
// The same on the 2-bit key cache, and its quantizer (score_q2.cu).
cudaError_t launch_anchor_score_q2(const ScoreArgs &a, int num_sms, cudaStream_t s);
cudaError_t launch_quantize_keys(const void *k, const int32_t *len, int B, int Hkv, int d, int Lmax,
                                 int start, void *kq, DevStatus *st, cudaStream_t s);

cudaError_t launch_refine_rescore(const ScoreArgs &a, cudaStream_t s);

struct CanonArgs {
    const int32_t *idx;        // [rows][kappa], any order, duplicates, -1 padding
    const int32_t *len;
    int B, Hkv, Lmax, kappa, radius;
    int32_t *out;              // [rows][kappa] canonical: ascending, distinct, -1 padded
    int32_t *out_off;          // nullable: [rows][kappa + 1] its proposal enumeration offsets
    DevStatus *st;
};
cudaError_t launch_canonicalize(const CanonArgs &a, cudaStream_t s);

struct SelectArgs {
    const float *S;            // anchor: [rows][Lmax] scores by position; refine: candidate scores
    const int32_t *cpos;       // refine: [rows][Lmax] candidate positions; nullptr for the anchor
    const int32_t *src_off;    // refine: [rows][src_kappa + 1]; its last entry = number of candidates
    const int32_t *len;
    int B, Hkv, Lmax, kappa, radius;
    int src_kappa;             // refine: entries of the source selection (0: kappa)
    int n_bound;               // bound on a row's items, sizes the cluster (0: from kappa, radius)
    int keep_hist;             // nonzero: leave the histogram for another selection of the same scores
    // refine: nz selections in one launch (grid z), selection z reading S, cpos,
    // hist, cspill shifted by z times the strides below and writing outz[z]
    // (nz > 1; idx_out otherwise); cstride is the row stride of S, cpos and
    // the two halves of cspill (0: Lmax)
    int nz;
    int cstride;
    size_t zS, zhist, zspill;
    int32_t *outz[8];
    uint32_t *hist;            // [rows][kHistBins], left zeroed (unless keep_hist)
    uint64_t *cspill;          // [rows][2][Lmax] overflow of the CTAs' candidate and tie lists
    int32_t *idx_out;          // [rows][kappa]
    int32_t *prop_off;         // nullable: [rows][kappa + 1] offsets of the next proposal
    DevStatus *st;
    uint64_t wait_ns;          // bound on the wait for the slice copies
    int row_cap;               // one-block-per-row kernel: bound on a row's items (set by the launcher)
};
cudaError_t launch_select(const SelectArgs &a, cudaStream_t s);

// Selection of a refined layer from the rescoring's runs (select_row.cu): one
// block per row (and per batched layer z); the selection leaves as ascending
// positions, -1 padded.
struct RunSelectArgs {
    const uint64_t *runs;      // [rows][nruns][kRunCap]
    const int32_t *run_cnt;    // [rows][nruns]
    int nruns;
    uint32_t *hist;            // [rows][kHistBins], left zeroed
    const int32_t *len;
    int B, Hkv, Lmax, kappa;
    uint64_t *tie_spill;       // [rows][tie_cap] overflow of the first-digit ties
    int tie_cap;
    int nz;                    // z > 0: shifted by z * zruns, z * zcnt, z * zhist, z * ztie
    size_t zruns, zcnt, zhist, ztie;
    int32_t *outz[8];          // nz > 1: layer z's selection; else idx_out
    int32_t *idx_out;          // [rows][kappa]
    DevStatus *st;
};
cudaError_t launch_select_runs(const RunSelectArgs &a, cudaStream_t s);
// One block per row (select_row.cu), for rows of at most kRowMaxItems items
// and budgets of at most kRowMaxKappa.
constexpr int kRowMaxItems = 1 << 18;
constexpr int kRowMaxKappa = 8192;
bool select_row_fits(int items, int kappa);
cudaError_t launch_select_row(const SelectArgs &a, int items, cudaStream_t s);

struct AttnArgs {
    const void *q;             // bf16 [B][Hq][d]
    const void *k, *v;         // bf16 [B][Hkv][Lmax][d]
    const int32_t *len;
    const int32_t *idx;        // [rows][idx_stride]
    int idx_stride, n_idx;
    int B, Hkv, G, d, Lmax;
    float scale;
    float *part_acc;           // [rows][nsplit][G][d]
    float *part_ml;            // [rows][nsplit][G][2]
    RowCtl *ctl;
    void *out;                 // bf16 [B][Hq][d]
    // nullable: instead of out, the row's merged split softmax unnormalised,
    // [B*Hq][d + 2] fp32 = (sum_s e^(m_s - M) acc_s, M, sum_s e^(m_s - M) l_s),
    // the partial of one context-parallel rank
    float *cp_part;
    DevStatus *st;
};
constexpr int kAttnChunk = 64;
cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t s);

// Static scratch of the no-workspace attention variant (attn_static.cu).
constexpr int kStaticAttnMaxRows = 1024;                 // B * Hkv
constexpr size_t kStaticAttnMaxAccFloats = (size_t)1 << 20;   // rows * splits * G * d
struct StaticAttnScratch {
    DevStatus *st;
    RowCtl *ctl;
    float *part_ml, *part_acc;
};
cudaError_t static_attn_scratch(StaticAttnScratch *out);

// Diagnostic export of a refined layer's candidates (misc.cu): the proposal
// of the canonical source `src` ([rows][E], radius r) in ascending order, with
// the scores the rescoring left by position in Spos (row stride Lmax).
cudaError_t launch_export_candidates(const int32_t *src, int E, int radius, const int32_t *len,
                                     int B, int Hkv, int Lmax, const float *Spos,
                                     int32_t *cand_pos, float *cand_score, int32_t *cand_count,
                                     int cand_cap, DevStatus *st, cudaStream_t s);

cudaError_t launch_debug_wait(DevStatus *st, uint64_t limit_ns, cudaStream_t s);

}  // namespace prism
