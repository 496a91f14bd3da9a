// quantize.cu -- HBM-bound MXFP4 quantize/pack kernels for sm_100a.
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
// Quantization for MXFP4 Attention", abstract -- MXFP4 operands with
// power-of-two microscaling; scale rule OCP (floor(log2 amax) - 2) or UOS
// (smallest e with amax <= Qmax * 2^e, Qmax = 7.25).
//
//  * quantize_rows_kernel: blocks of 32 consecutive elements of a row (the
//    standalone op).  Each thread loads 16 bytes (8 bf16), a quad of
//    lanes owns one block: the block maximum is an integer max over |bf16|
//    bit patterns plus two xor-shuffles, the exponent comes from the maximum's
//    exponent and mantissa fields, the 8 scaled values go through four
//    cvt.rn.satfinite.e2m1x2 and leave as one 32-bit store.  The quad's first
//    lane stores the E8M0 byte (row-major scales).
//  * quantize_vt_kernel: V blocks of 32 consecutive tokens per channel,
//    written transposed (V^T, tokens contiguous): a CTA stages 128 tokens x d
//    channels in shared memory and each thread quantizes the blocks of a pair
//    of channels over a run of tokens from there (one 32-bit shared-memory
//    read per token for both channels), row-major scales.
//  * regroup_sf_kernel: row-major scales -> the 128-row regrouped order.
// The forward's own preparation (regrouped scales, one launch) is prepare.cu.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "mxfp4_block.cuh"
#include "ptx.cuh"

namespace mxattn {

namespace {

constexpr int kQuantThreads = 256;
#ifndef MXATTN_QUANT_UNROLL
#define MXATTN_QUANT_UNROLL 8
#endif
#ifndef MXATTN_QUANT_CTAS_PER_SM
#define MXATTN_QUANT_CTAS_PER_SM 8
#endif
constexpr int kUnroll = MXATTN_QUANT_UNROLL;             // 16-byte loads in flight per lane
constexpr int kCtasPerSm = MXATTN_QUANT_CTAS_PER_SM;     // grid of the grid-stride quantizer

// Row quantization with row-major scales [rows, cols/32] (the standalone op):
// grid-stride over 16-byte chunks, kUnroll loads in flight per lane.
__global__ void __launch_bounds__(kQuantThreads) quantize_rows_kernel(const uint16_t* __restrict__ x,
                                                                      uint32_t* __restrict__ codes,
                                                                      uint8_t* __restrict__ scales, int64_t n_chunks,
                                                                      uint32_t sf_thresh, uint32_t* status) {
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
    for (int64_t base = warp * (32 * kUnroll); base < n_chunks; base += n_warps * (32 * kUnroll)) {
        uint4 raw[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * 32 + lane;
            raw[u] = (i < n_chunks) ? __ldcs(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * 32 + lane;
            int e;
            const uint32_t packed = quantize_quad_bf16(raw[u], sf_thresh, e);
            if (i < n_chunks) {
                codes[i] = packed;
                if ((lane & 3) == 0) scales[i >> 2] = static_cast<uint8_t>(e + 127);
            }
        }
    }
}

// V^T quantization: grid (G token groups of 128, BH), 128 threads.  The CTA
// stages 128 tokens x D channels (bf16) in shared memory.  Each thread then
// owns a pair of adjacent channels over a run of 256 / D * 16 tokens (64 for
// D = 128, 32 for D = 64): it reads its two channels of a token as one 32-bit
// word (a warp reads 128 contiguous bytes of a token row), quantizes the 32-
// token blocks of both channels, and writes each channel's codes for its run
// as contiguous 16-byte stores.
template <int D>
__global__ void __launch_bounds__(128) quantize_vt_kernel(const uint16_t* __restrict__ v, int N, int npad, uint32_t sf_thresh,
                                                          uint8_t* __restrict__ codes_t, uint8_t* __restrict__ scales_t) {
    constexpr int kPairs = D / 2;             // channel pairs
    constexpr int kRuns = 128 / kPairs;       // token runs per 128-token group (2 or 4)
    constexpr int kRun = 128 / kRuns;         // tokens per run (64 or 32)
    constexpr int kBlocks = kRun / 32;        // 32-token blocks per run (2 or 1)
    __shared__ __align__(16) uint16_t tile[128 * D];
    const int g = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int t0 = g * 128;
    const int tid = threadIdx.x;
    constexpr int kChunksPerRow = D / 8;
    constexpr int kPerThread = 128 * kChunksPerRow / 128;  // 16-byte loads in flight per thread
    uint4 val[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int c = tid + u * 128;
        const int t = c / kChunksPerRow;
        val[u] = (t0 + t < N) ? __ldcs(reinterpret_cast<const uint4*>(v + (bh * N + t0 + t) * D) + (c % kChunksPerRow))
                              : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) reinterpret_cast<uint4*>(tile)[tid + u * 128] = val[u];
    __syncthreads();
    const int cp = tid % kPairs;   // channels 2 cp, 2 cp + 1
    const int run = tid / kPairs;  // tokens [run * kRun, run * kRun + kRun) of the group
    const uint32_t* tile32 = reinterpret_cast<const uint32_t*>(tile);
#pragma unroll
    for (int b = 0; b < kBlocks; ++b) {
        uint32_t raw[32];  // token i of the block: channel 2 cp in the low half, 2 cp + 1 in the high half
#pragma unroll
        for (int i = 0; i < 32; ++i) raw[i] = tile32[(run * kRun + 32 * b + i) * kPairs + cp];
        uint32_t words[2][4];
        int e[2];
        quantize_vt_block_bf16(raw, sf_thresh, words, e);
        const int tb = t0 + run * kRun + 32 * b;  // first token of the block
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int ch = 2 * cp + h;
            uint8_t* rowp = codes_t + (bh * D + ch) * static_cast<int64_t>(npad / 2);
            if (tb < npad) {
                *reinterpret_cast<uint4*>(rowp + tb / 2) = make_uint4(words[h][0], words[h][1], words[h][2], words[h][3]);
                scales_t[(bh * D + ch) * static_cast<int64_t>(npad / 32) + tb / 32] = static_cast<uint8_t>(e[h] + 127);
            }
        }
    }
}

// Row-major scales -> regrouped scales for Q, K (blocks along d) and V^T
// (blocks along tokens), one byte per thread; also clears the status word.
__global__ void __launch_bounds__(kQuantThreads) regroup_sf_kernel(const uint8_t* __restrict__ q_scales,
                                                                   const uint8_t* __restrict__ k_scales,
                                                                   const uint8_t* __restrict__ vt_scales, int64_t BH,
                                                                   int N, int d, int groups, uint8_t* __restrict__ q_sf,
                                                                   uint8_t* __restrict__ k_sf,
                                                                   uint8_t* __restrict__ v_sf, uint32_t* status) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    const int64_t per = BH * groups * 512;
    const int npad32 = (N + 31) / 32;
    const int kb = d / 32;
    for (int64_t o = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x; o < per;
         o += static_cast<int64_t>(gridDim.x) * kQuantThreads) {
        const int64_t chunk = o / 512;
        const int pos = static_cast<int>(o % 512);
        const int64_t bh = chunk / groups;
        const int g = static_cast<int>(chunk % groups);
        const int m = (pos / 16) + 32 * ((pos % 16) / 4);
        const int k = pos % 4;
        const int r = g * 128 + m;
        uint8_t qv = 0, kv = 0, vv;
        if (r < N && k < kb) {
            qv = q_scales[(bh * N + r) * kb + k];
            kv = k_scales[(bh * N + r) * kb + k];
        }
        if (m < d) {
            const int tb = 4 * g + k;
            vv = (tb < npad32) ? vt_scales[(bh * d + m) * static_cast<int64_t>(npad32) + tb] : 0;
        } else {
            vv = 127;
        }
        q_sf[o] = qv;
        k_sf[o] = kv;
        v_sf[o] = vv;
    }
}

int grid_for(int64_t work_items, int per_block) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (work_items + per_block - 1) / per_block;
    const int64_t cap = static_cast<int64_t>(sms) * kCtasPerSm;
    return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_quantize_rows(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows, int cols,
                                 uint32_t sf_thresh, uint32_t* status, cudaStream_t stream) {
    const int64_t n_chunks = rows * cols / 8;
    quantize_rows_kernel<<<grid_for(n_chunks / kUnroll, kQuantThreads), kQuantThreads, 0, stream>>>(
        static_cast<const uint16_t*>(x), reinterpret_cast<uint32_t*>(codes), scales, n_chunks, sf_thresh, status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_vt(const void* v, int64_t BH, int N, int d, uint32_t sf_thresh, uint8_t* codes_t,
                               uint8_t* scales_t, cudaStream_t stream) {
    const int npad = (N + 31) / 32 * 32;
    dim3 grid((N + 127) / 128, static_cast<unsigned>(BH));
    if (d == 128)
        quantize_vt_kernel<128><<<grid, 128, 0, stream>>>(static_cast<const uint16_t*>(v), N, npad, sf_thresh, codes_t,
                                                           scales_t);
    else
        quantize_vt_kernel<64><<<grid, 128, 0, stream>>>(static_cast<const uint16_t*>(v), N, npad, sf_thresh, codes_t,
                                                          scales_t);
    return cudaGetLastError();
}

cudaError_t launch_regroup_sf(const uint8_t* q_scales, const uint8_t* k_scales, const uint8_t* vt_scales, int64_t BH,
                              int N, int d, int groups, uint8_t* q_sf, uint8_t* k_sf, uint8_t* v_sf,
                              uint32_t* status, cudaStream_t stream) {
    const int64_t per = BH * groups * 512;
    regroup_sf_kernel<<<grid_for(per, kQuantThreads), kQuantThreads, 0, stream>>>(
        q_scales, k_scales, vt_scales, BH, N, d, groups, q_sf, k_sf, v_sf, status);
    return cudaGetLastError();
}

}  // namespace mxattn
