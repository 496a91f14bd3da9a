// noalloc.cu -- mxattn_forward_noalloc: mxattn_forward with library-owned scratch.
//
// Some callers cannot hand the library a workspace they allocated: code
// embedded in a host framework that owns all device memory through its own
// pool and forbids raw cudaMalloc, or a latency-critical loop that must not
// pay for cudaMalloc's implicit device synchronization.  For them this entry
// point keeps its scratch in a fixed-size array in device memory that is part
// of this library's CUDA module: it is created when the module is loaded on a
// device and lives until the process exits.  No call here allocates or frees
// device memory.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "mxattn.h"

#define MXATTN_API extern "C" __attribute__((visibility("default")))

namespace {

// Largest workspace this entry point can serve (mxattn_workspace_size bytes).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

// The scratch itself.  In host code `g_noalloc_scratch` is only a handle for
// the runtime; the device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the first call on a device does this set-up).
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

MXATTN_API mxattn_status mxattn_forward_noalloc(const void* Q, const void* K, const void* V, int B, int H, int N,
                                                int d, int kv_tile, int pnq, mxattn_rule rule, float softmax_scale,
                                                float* O, mxattn_stream_t stream) {
    const size_t need = mxattn_workspace_size(B, H, N, d);
    if (need == 0) return (d != 64 && d != 128) ? MXATTN_ERR_UNSUPPORTED : MXATTN_ERR_INVALID;
    if (need > kNoAllocScratchBytes) return MXATTN_ERR_UNSUPPORTED;  // shape too large for the fixed scratch
    void* scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return MXATTN_ERR_CUDA;
    // The quantize kernels rewrite every workspace byte the attention kernel
    // reads and reset the status word, so stale contents of the previous call
    // do not leak into this one.
    return mxattn_forward(Q, K, V, B, H, N, d, kv_tile, pnq, rule, softmax_scale, O, scratch, kNoAllocScratchBytes,
                          stream);
}
