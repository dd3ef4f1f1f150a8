// attn_static.cu -- device scratch of the no-workspace variant of the sparse
// decode attention (prism_sparse_decode_noalloc).
//
// Some callers cannot hand the library device scratch: a host that holds only
// device pointers to its KV cache and has no device allocator of its own, or
// one that must not allocate device memory once it has started.  For them the
// split-K partials and the per-row merge counters live in this file-scope
// device array, sized for a stated maximum (see include/prism.h).  Nothing here
// allocates: the array exists for as long as the library is loaded.
//
// The first use on a device (and again the first use after that device's
// context was replaced, e.g. by cudaDeviceReset, when the module may load at
// another address) looks up the array's address (cudaGetSymbolAddress) and
// caches it with the context's unique id; that first call should therefore
// come before any stream capture.  Every call shares the one array, so calls
// that overlap in time (on different streams or threads) race on it.
#include <mutex>

#include "prism_internal.cuh"

namespace prism {

namespace {

constexpr size_t kStatusBytes = 256;
constexpr size_t kCtlBytes = (size_t)kStaticAttnMaxRows * sizeof(RowCtl);
constexpr size_t kMlFloats = 2 * (kStaticAttnMaxAccFloats / 64);     // 2 per (row, split, head), d >= 64
constexpr size_t kCtlOff = kStatusBytes;
constexpr size_t kMlOff = kCtlOff + ((kCtlBytes + 255) & ~(size_t)255);
constexpr size_t kAccOff = kMlOff + ((kMlFloats * 4 + 255) & ~(size_t)255);
constexpr size_t kScratchBytes = kAccOff + kStaticAttnMaxAccFloats * 4;

static __device__ __align__(256) uint8_t g_attn_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t *g_base[kMaxDevices] = {};
unsigned long long g_ctx[kMaxDevices] = {};

// Unique id of the calling thread's current context (0 if the driver cannot
// tell), through the driver entry points the runtime exposes.
unsigned long long current_context_id() {
    using GetCurrent = int (*)(void **);
    using GetId = int (*)(void *, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {            // under g_mu
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrent>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
        looked_up = true;
    }
    void *ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == 0 && ctx && get_id(ctx, &id) == 0) return id;
    return 0;
}

}  // namespace

cudaError_t static_attn_scratch(StaticAttnScratch *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_base[dev] || (ctx != 0 && ctx != g_ctx[dev])) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess) return e;
        g_base[dev] = static_cast<uint8_t *>(p);
        g_ctx[dev] = ctx;
    }
    uint8_t *b = g_base[dev];
    out->st = reinterpret_cast<DevStatus *>(b);
    out->ctl = reinterpret_cast<RowCtl *>(b + kCtlOff);
    out->part_ml = reinterpret_cast<float *>(b + kMlOff);
    out->part_acc = reinterpret_cast<float *>(b + kAccOff);
    return cudaSuccess;
}

}  // namespace prism
