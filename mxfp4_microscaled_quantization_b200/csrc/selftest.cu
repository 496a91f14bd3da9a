// selftest.cu -- mxattn_wait_selftest: drives the attention kernel's bounded
// mbarrier wait to its time limit on purpose, so that a caller can check that
// a wait which is never satisfied ends, reports MXATTN_ERR_TIMEOUT and leaves
// the CUDA context usable.  Nothing here faults or traps: the kernel waits on
// an mbarrier that nobody arrives at (unless asked to arrive) and returns.
#include <cuda_runtime.h>

#include <cstdint>

#include "mxattn.h"
#include "ptx.cuh"

#define MXATTN_API extern "C" __attribute__((visibility("default")))

namespace mxattn {
namespace {

constexpr uint32_t kTimeoutCode = 4u;  // MXATTN_ERR_TIMEOUT

// One warp.  out[0] <- 0 or kTimeoutCode, out[1] <- microseconds spent in the
// wait, out[2] <- bit 0: the abort flag was raised, bit 1: the
// warp left the wait without the barrier completing.
__global__ void __launch_bounds__(32) wait_selftest_kernel(int arrive, uint64_t timeout_ns, uint32_t* out) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        out[0] = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && arrive) mbar_arrive(&bar);
    __syncwarp();
    const uint64_t t0 = global_timer_ns();
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bar, 0, &abort_flag, out, kTimeoutCode, timeout_ns));
    const uint64_t t1 = global_timer_ns();
    __syncwarp();
    if (threadIdx.x == 0) {
        out[1] = static_cast<uint32_t>((t1 - t0) / 1000u);
        out[2] = (abort_flag ? 1u : 0u) | (ok ? 0u : 2u);
    }
}

}  // namespace
}  // namespace mxattn

MXATTN_API mxattn_status mxattn_wait_selftest(int arrive, unsigned timeout_us, unsigned* out, mxattn_stream_t stream) {
    if (out == nullptr || timeout_us == 0 || timeout_us > 1000000u) return MXATTN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(out) & 3u) != 0) return MXATTN_ERR_INVALID;
    mxattn::wait_selftest_kernel<<<1, 32, 0, stream>>>(arrive, uint64_t(timeout_us) * 1000u, out);
    return cudaGetLastError() == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}
