// arkv_reassign_noalloc: the tier reassignment with its scratch memory in a
// file-scope device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they reassign:
// code that runs while a CUDA graph is being captured (cudaMalloc is not a
// stream operation that a capture can record), serving engines that reserve all
// device memory up front and forbid any later allocation, and plugins hosted by
// a framework that owns the device allocator.  For them this entry point takes
// no workspace at all and allocates nothing: its scratch (the per-row slot lists
// of the compaction and, for rows too long for shared memory, the score keys)
// lives in g_noalloc_scratch below.
//
// The array is a module global, so every GPU that loads this library holds
// ARKV_NOALLOC_SCRATCH_BYTES of it until the process exits (or its context is
// destroyed, after which the next call finds the array's new address).  All calls share it
// and it keeps whatever the last call left; the kernel writes every scratch word
// before it reads it, so nothing needs clearing.  Calls whose executions overlap
// on the GPU (different streams, or different layers without ordering) race on
// the array and must be serialised by the caller.
#include <stdio.h>

#include <mutex>

#include <cudaTypedefs.h>

#include "arkv_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ARKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];   // id of the context the address belongs to
bool g_scratch_set[kMaxDevices];

// Unique id of the calling thread's current CUDA context (driver entry points,
// looked up once), or 0 if it cannot be had.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx) get_id(ctx, &id);
    return id;
}

// The device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side handle, so the address is looked up with
// the device current (cudaGetSymbolAddress) the first time, and again whenever
// the device's context has changed since (the module, and with it the array, is
// reloaded in a new context).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_scratch_set[dev] || (ctx != 0 && ctx != g_scratch_ctx[dev])) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = current_context_id();   // the lookup made the context current if it was not
        g_scratch_set[dev] = true;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int arkv_reassign_noalloc(const arkv_cfg* cfg, int32_t step, float r, const int32_t* ctx_len,
                                     arkv_layer_cache* cache, uint8_t* tier_dbg, arkv_stream_t stream) {
    const size_t need = arkv_workspace_bytes(cfg, ARKV_WS_REASSIGN, 0);
    if (need == 0) {
        if (!cfg) arkv::set_last_error("arkv_reassign_noalloc: cfg is null");
        return ARKV_EINVAL;   // the configuration check has described the problem
    }
    if (need > (size_t)ARKV_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "arkv_reassign_noalloc: this layer needs %zu bytes of scratch, more than the "
                 "built-in %u; use arkv_reassign with a workspace",
                 need, (unsigned)ARKV_NOALLOC_SCRATCH_BYTES);
        arkv::set_last_error(msg);
        return ARKV_EINVAL;
    }
    void* scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "arkv_reassign_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        arkv::set_last_error(msg);
        return ARKV_ECUDA;
    }
    return arkv_reassign(cfg, step, r, ctx_len, cache, tier_dbg, scratch, need, stream);
}
