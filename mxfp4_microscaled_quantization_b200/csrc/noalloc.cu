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
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kernels.cuh"
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
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context id the address belongs to (0: none yet)

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Driver entry points looked up through the runtime (no link-time dependency on libcuda).
void* driver_fn(const char* name) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return fn;
}

// Id of the current context: unique for the life of the process, so a context
// created after cudaDeviceReset has a different id from the one it replaces.
cudaError_t current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
    static CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
    if (get_current == nullptr || get_id == nullptr) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    return get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of the scratch array in the current device's current
// context.  The first call in a context looks it up (this is the set-up step:
// it runs with that device current); later calls reuse the cached address
// while the same context is current.
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    unsigned long long ctx = 0;
    e = current_context_id(&ctx);
    if (e == cudaErrorDeviceUninitialized) {
        // No context is current yet: cudaSetDevice makes the device's primary context current.
        e = cudaSetDevice(dev);
        if (e != cudaSuccess) return e;
        e = current_context_id(&ctx);
    }
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

MXATTN_API mxattn_status mxattn_forward_noalloc(const void* Q, const void* K, const void* V, int B, int H, int N,
                                                int d, int kv_tile, int pnq, mxattn_rule rule, float softmax_scale,
                                                float* O, mxattn_stream_t stream) {
    // The same argument checks, in the same order, as mxattn_forward; then the scratch's limit.
    if (rule != MXATTN_RULE_OCP && rule != MXATTN_RULE_UOS) return MXATTN_ERR_INVALID;
    const mxattn_status st = mxattn::check_attention_shape(B, H, N, d, kv_tile, pnq, O);
    if (st != MXATTN_OK) return st;
    const size_t need = mxattn_workspace_size(B, H, N, d);
    if (need == 0) return MXATTN_ERR_INVALID;
    if (need > kNoAllocScratchBytes) return MXATTN_ERR_UNSUPPORTED;  // shape too large for the fixed scratch
    void* scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return MXATTN_ERR_CUDA;
    // The preparation kernel rewrites every workspace byte the attention kernel
    // reads and resets the status word, so stale contents of the previous call
    // do not leak into this one.
    return mxattn_forward(Q, K, V, B, H, N, d, kv_tile, pnq, rule, softmax_scale, O, scratch, kNoAllocScratchBytes,
                          stream);
}
