// selftest.cu -- self-tests of pieces of the attention kernel.
//
// mxattn_wait_selftest drives the kernel's bounded mbarrier wait to its time
// limit on purpose, so that a caller can check that a wait which is never
// satisfied ends, reports MXATTN_ERR_TIMEOUT and leaves the CUDA context
// usable.  Nothing here faults or traps: the kernel waits on an mbarrier that
// nobody arrives at (unless asked to arrive) and returns.
//
// mxattn_p_selftest runs the softmax's decisions on P -- E2M1 codes of the
// exponentials on each of the three exponential paths, the MXFP4 block
// exponent and the NVFP4 block scale -- on caller inputs, through the same
// device functions the attention kernel uses, so they can be compared with
// the CPU oracle directly.
#include <cuda_runtime.h>

#include <cmath>
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

// The softmax's P decisions on a list of inputs, through the same device
// functions the attention kernel calls (8 inputs per thread, grid-stride).
//   path 0/1/2: in = w, out = E2M1 code of 2^w by ex2.approx / the FMA-pipe
//               code-only stand-in / the FMA-pipe degree-5 exponential, each
//               followed by cvt.rn.satfinite.e2m1x2;
//   path 3:     in = x (log2 of a block's largest exponential), out = the
//               MXFP4 block exponent for the scale boundary (OCP, or log2 Qmax);
//   path 4:     in = x, out = the NVFP4 block scale byte (E4M3 of 2^x * 448);
//   path 5:     in = v, out = E2M1 code of v itself (the rounding step alone).
__global__ void __launch_bounds__(256) p_selftest_kernel(int path, const float* __restrict__ in, int64_t n8,
                                                         int ocp, float log2q, int32_t* __restrict__ out) {
    for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < n8;
         g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = in[8 * g + i];
        if (path <= 2 || path == 5) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                if (path == 5) {
                    f[i] = v[i];
                    f[i + 1] = v[i + 1];
                } else if (path == 0) {
                    f[i] = ex2_approx(v[i]);
                    f[i + 1] = ex2_approx(v[i + 1]);
                } else if (path == 1) {
                    exp2_code_sat_x2(v[i], v[i + 1], 0.125f, 0.25f, f[i], f[i + 1]);  // u = (w + 2) / 8
                } else {
                    exp2_fma_x2(v[i], v[i + 1], f[i], f[i + 1]);
                }
            }
            const uint32_t codes = pack_e2m1x8(f);
#pragma unroll
            for (int i = 0; i < 8; ++i) out[8 * g + i] = static_cast<int32_t>((codes >> (4 * i)) & 0xFu);
        } else if (path == 3) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t byte;
                const float e = ocp ? p_block_exp<true>(v[i], 1.f, 0.f, byte) : p_block_exp<false>(v[i], 1.f, log2q, byte);
                out[8 * g + i] = static_cast<int32_t>(e);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) out[8 * g + i] = static_cast<int32_t>(nv_p_block_scale(v[i]));
        }
    }
}

}  // namespace
}  // namespace mxattn

MXATTN_API mxattn_status mxattn_p_selftest(int path, const float* in, int64_t n, float qmax, int32_t* out,
                                           mxattn_stream_t stream) {
    if (path < 0 || path > 5 || n < 0 || n % 8 != 0) return MXATTN_ERR_INVALID;
    if (path == 3 && !(qmax > 4.f && qmax <= 8.f)) return MXATTN_ERR_INVALID;
    if (n == 0) return MXATTN_OK;
    if (in == nullptr || out == nullptr || (reinterpret_cast<uintptr_t>(in) & 3u) || (reinterpret_cast<uintptr_t>(out) & 3u))
        return MXATTN_ERR_INVALID;
    const bool ocp = qmax >= 8.f;
    const float log2q = ocp ? 0.f : static_cast<float>(std::log2(static_cast<double>(qmax)));
    const int64_t n8 = n / 8;
    const int grid = static_cast<int>(n8 / 256 + 1 < 4096 ? n8 / 256 + 1 : 4096);
    mxattn::p_selftest_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(path, in, n8, ocp ? 1 : 0,
                                                                                         log2q, out);
    return cudaGetLastError() == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_wait_selftest(int arrive, unsigned timeout_us, unsigned* out, mxattn_stream_t stream) {
    if (out == nullptr || timeout_us == 0 || timeout_us > 1000000u) return MXATTN_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(out) & 3u) != 0) return MXATTN_ERR_INVALID;
    mxattn::wait_selftest_kernel<<<1, 32, 0, stream>>>(arrive, uint64_t(timeout_us) * 1000u, out);
    return cudaGetLastError() == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}
