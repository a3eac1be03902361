// lm_mlp_noalloc.cu -- the relu^2 MLP backward for callers that cannot
// allocate device memory.
//
// lm_relu2_mlp_bwd needs a caller-provided scratch workspace (the GEMMs'
// split-K scratch, the e5m2 codes of dY and dH, the bf16 dH and two scale
// blocks).  Some callers have no way to provide one: plugins whose host
// framework owns the whole device memory pool and forbids allocation in its
// execute callback, and latency-critical loops that cannot afford the
// device-wide synchronisation that cudaMalloc/cudaFree may cause.  For them
// this file keeps the workspace in a fixed device array that the library owns.
//
// Limits and sharing:
//  - the array holds kScratchBytes (64 MiB); shapes whose workspace
//    (lm_relu2_mlp_workspace_size) is larger are rejected with
//    LM_ERR_UNSUPPORTED_SHAPE before anything is enqueued;
//  - every GPU that loads this part of the library keeps the array until
//    the process exits;
//  - all calls on a device share the one array: two calls whose work
//    overlaps on the GPU (different streams, no ordering between them) race
//    and corrupt each other's results.  Calls on one stream are safe;
//  - the array keeps whatever the previous call left in it; the backward
//    zeroes what must start at zero (its amax accumulators and the split-K
//    flags) on every call.
#include <atomic>

#include "lm_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;

// Library-owned scratch, one instance per device.  In host code the name is
// only a handle for cudaGetSymbolAddress, never a device address.
static __device__ __align__(256) unsigned char g_mlp_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
// Device address of the array per device, looked up on the first call made
// with that device current.  Host threads may race on the first lookup; each
// stores the same address, and the atomics keep that well defined.  The
// address is not valid after cudaDeviceReset on that device.
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch on the current device.  nullptr on failure.
void* scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    if (cudaGetSymbolAddress(&p, g_mlp_bwd_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev].store(p, std::memory_order_release);
    return p;
}

}  // namespace

extern "C" lm_status lm_relu2_mlp_bwd_noalloc(const void* dY, const lm_mlp_saved* saved,
                                              int64_t M, int64_t d, int64_t f, void* dX,
                                              void* dW_up, void* dW_down, lm_stream_t stream) {
    const size_t need = lm_relu2_mlp_workspace_size(M, d, f);
    if (need == 0 || need > kScratchBytes) return LM_ERR_UNSUPPORTED_SHAPE;
    void* ws = scratch_address();
    if (!ws) return LM_ERR_CUDA;
    return lm_relu2_mlp_bwd(dY, saved, M, d, f, dX, dW_up, dW_down, ws, kScratchBytes, stream);
}

extern "C" size_t lm_relu2_mlp_bwd_noalloc_max_bytes(void) { return kScratchBytes; }
