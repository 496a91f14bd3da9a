// mma_peak.cu -- the throughput ceiling of the attention kernel's tensor-core
// instruction on this GPU (a measurement utility; the method itself has no
// counterpart).
//
// Each CTA keeps one 128 x 128 fp32 accumulator in TMEM and has one thread
// issue tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 back to back
// with M = 128, N = 128, K = 64 -- the shape and the shared-memory / scale-
// factor descriptors of the attention kernel's S = Q K^T product -- on
// operands that stay in shared memory, so nothing but the tensor core is
// timed.  The operands are a fixed mix of E2M1 codes with unit scales; the
// result is never read.  The one wait (for the final commit) is bounded like
// every wait in the library.  Each CTA also records the SM clock cycles from
// its first issue to the completion of its last MMA, so the rate can be
// stated per clock, independent of the clock the power cap allows.
#include <cuda_runtime.h>

#include <cstdint>

#include "mxattn.h"
#include "ptx.cuh"

#define MXATTN_API extern "C" __attribute__((visibility("default")))

namespace mxattn {
namespace {

constexpr uint64_t kLoopTimeoutNs = 2000000000ull;  // 2 s; a full launch takes milliseconds
constexpr uint32_t kTimeoutCode = 4u;               // MXATTN_ERR_TIMEOUT
constexpr int kThreads = 128;
constexpr int kSmemBytes = 16384 + 1024 + 1024;     // A and B tiles, two scale atoms, alignment slack

__device__ __forceinline__ uint64_t atom_desc(const void* p) {
    // 32 rows x 16 bytes, rows contiguous: core matrices of 8 rows 128 bytes apart
    return smem_desc(smem_u32(p), 0, 128, kLayoutNone);
}

__global__ void __launch_bounds__(kThreads) mxf4_mma_loop_kernel(int iters, uint32_t* status,
                                                                  unsigned long long* cycles) {
    extern __shared__ uint8_t smem_raw[];
    // Aligned by an offset from the shared array itself, so every derived pointer
    // keeps the shared address space (32-bit addressing, nothing held as a generic pointer).
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;           // 128 rows x 64 bytes (K = 128 E2M1 values), 64-byte swizzle
    uint8_t* sB = smem + 8192;    // the same for B
    uint8_t* sSf = smem + 16384;  // scale atoms of A and B (512 bytes each)
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_holder;
    __shared__ int abort_flag;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    for (int i = tid; i < 16384 / 4; i += kThreads)
        reinterpret_cast<uint32_t*>(smem)[i] = (0x9E3779B9u * static_cast<uint32_t>(i + 1)) & 0x77777777u;
    for (int i = tid; i < 256; i += kThreads) reinterpret_cast<uint32_t*>(sSf)[i] = 0x7F7F7F7Fu;  // 2^0
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbarrier_init();
    }
    fence_proxy_async_smem();
    if (warp == 0) {
        tmem_alloc(&tmem_holder, 256);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = tmem_holder;
    if (warp == 0) {
        const bool leader = elect_one_sync();
        unsigned long long t0 = 0;
        if (leader) {
            t0 = clock64();
            tc_cp_sf(tbase + 128, atom_desc(sSf));
            tc_cp_sf(tbase + 132, atom_desc(sSf + 512));
            const uint64_t adesc = smem_desc(smem_u32(sA), 16, 512, kLayoutSw64);
            const uint64_t bdesc = smem_desc(smem_u32(sB), 16, 512, kLayoutSw64);
            for (int it = 0; it < iters; ++it) {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    tc_mma_mxf4(tbase, adesc + 2 * kk, bdesc + 2 * kk, mxf4_idesc(128, 2 * kk, 2 * kk), tbase + 128,
                                tbase + 132, (it > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&bar);
        }
        __syncwarp();
        mbar_wait_bounded(&bar, 0, &abort_flag, status, kTimeoutCode, kLoopTimeoutNs);
        if (leader && cycles != nullptr) cycles[blockIdx.x] = clock64() - t0;
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tbase, 256);
    }
}

}  // namespace
}  // namespace mxattn

MXATTN_API mxattn_status mxattn_mxf4_mma_loop(int ctas, int iters, uint32_t* status, uint64_t* cycles,
                                              mxattn_stream_t stream) {
    if (ctas < 1 || ctas > 4096 || iters < 1 || iters > 200000 || status == nullptr ||
        (reinterpret_cast<uintptr_t>(status) & 3u) || (reinterpret_cast<uintptr_t>(cycles) & 7u))
        return MXATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return MXATTN_ERR_CUDA;
    mxattn::mxf4_mma_loop_kernel<<<ctas, mxattn::kThreads, mxattn::kSmemBytes, s>>>(
        iters, status, reinterpret_cast<unsigned long long*>(cycles));
    return cudaGetLastError() == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}
