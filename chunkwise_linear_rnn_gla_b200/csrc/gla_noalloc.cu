// gla_fwd_noalloc: the forward pass for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: a
// plugin running under a host framework or inference server that owns every
// device allocation and gives plugins none, a latency-critical loop that must
// not risk the implicit device synchronisation cudaMalloc/cudaFree can cause,
// or a plain C caller with no device memory manager. For them this entry point
// runs the CUDA-core forward with its scratch in a fixed array that is part of
// the library image itself (a file-scope __device__ array), so nothing is
// allocated at call time: the caller still passes inputs and outputs.
//
// Costs and limits, stated once:
//  * Every GPU on which the library's kernels are loaded holds the array
//    (GLA_NOALLOC_SCRATCH_BYTES) until the process exits.
//  * Problems whose CUDA-core forward workspace exceeds the array are
//    rejected with GLA_ERR_WORKSPACE before anything is launched.
//  * All calls on a device share the one array, and it keeps what the last
//    call left in it. Every byte the kernels read is written earlier in the
//    same call (per-chunk cumsum, intra-chunk scores, per-chunk states), so
//    nothing needs clearing between calls; but calls whose execution overlaps
//    on the GPU (different streams, or different host threads) race on the
//    array and must be serialised by the caller.
//  * The device address of the array is looked up (cudaGetSymbolAddress) the
//    first time the entry point runs on each device, with that device
//    current, and looked up again if the device's context has changed since
//    (a device reset replaces the context and moves the array). That lookup
//    is host-side set-up and allocates nothing; make the first call on each
//    device, and the first call after a reset, before any stream capture
//    begins.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gla_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Per device: the context the address was looked up in (its process-unique id) and the address.
struct ScratchEntry {
    unsigned long long ctx_id;
    void* ptr;
};
ScratchEntry g_scratch[kMaxDevices] = {};

// The current context's process-unique id (cuCtxGetId), or 0 when none is current or the query is
// unavailable. A device reset destroys the primary context; the next context gets a new id, so an
// address looked up in the old one is never reused.
unsigned long long current_context_id() {
    static std::once_flag once;
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    });
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array in the current device's current context. Set-up (the symbol
// lookup) runs on the first call per device and again whenever the context has changed since (after
// a device reset); nullptr if the lookup failed.
void* scratch_on_current_device(gla_status* st) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = GLA_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_setup_mu);
    const unsigned long long id = current_context_id();
    ScratchEntry& e = g_scratch[dev];
    if (!e.ptr || id == 0 || id != e.ctx_id) {
        void* ptr = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (err != cudaSuccess || !ptr) {
            *st = GLA_ERR_CUDA;
            return nullptr;
        }
        // the lookup makes the device's primary context current if none was: take its id now
        e.ctx_id = id != 0 ? id : current_context_id();
        e.ptr = ptr;
    }
    *st = GLA_OK;
    return e.ptr;
}

}  // namespace

extern "C" gla_status gla_fwd_noalloc(const gla_desc* d, const void* q, const void* k, const void* v,
                                      const float* log_a, const float* h0, void* o, float* hT, void* stream) {
    if (!d) return GLA_ERR_INVALID_ARG;
    if (d->impl == GLA_IMPL_TC || d->state_mode == GLA_STATE_NONMATERIALIZED) return GLA_ERR_UNSUPPORTED;
    // Same descriptor, forced onto the CUDA-core path (the only one this
    // entry point runs), then the ordinary argument checks.
    gla_desc dd = *d;
    dd.impl = GLA_IMPL_SIMT;
    dd.flags = d->flags & GLA_FLAG_CHECKS;  // a forward has nothing to reuse
    const size_t need = gla_fwd_workspace_size(&dd);
    if (need == 0) {
        int32_t c = 0;
        const gla_status st = gla_resolve(&dd, &c, nullptr, nullptr, nullptr);
        return st == GLA_OK ? GLA_ERR_INVALID_ARG : st;
    }
    if (need > size_t(GLA_NOALLOC_SCRATCH_BYTES)) return GLA_ERR_WORKSPACE;
    if (!q || !k || !v || !log_a || !o) return GLA_ERR_INVALID_ARG;
    gla_status st = GLA_OK;
    void* scratch = scratch_on_current_device(&st);
    if (!scratch) return st;
    return gla_fwd(&dd, q, k, v, log_a, h0, o, hT, scratch, size_t(GLA_NOALLOC_SCRATCH_BYTES), stream);
}
