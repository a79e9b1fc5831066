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
// ARKV_NOALLOC_SCRATCH_BYTES of it until the process exits.  All calls share it
// and it keeps whatever the last call left; the kernel writes every scratch word
// before it reads it, so nothing needs clearing.  Calls whose executions overlap
// on the GPU (different streams, or different layers without ordering) race on
// the array and must be serialised by the caller.
#include <stdio.h>

#include <mutex>

#include "arkv_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ARKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];

// The device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side handle, so the address is looked up once
// per device (with that device current) and cached.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_scratch_once[dev], [dev] {
        void* p = nullptr;
        g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        g_scratch_ptr[dev] = p;
    });
    if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
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
