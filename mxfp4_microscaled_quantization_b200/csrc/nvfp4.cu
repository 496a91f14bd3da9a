// nvfp4.cu -- NVFP4 quantize kernels (the comparison variant) for sm_100a.
//
// The MXAttention abstract ("MXAttention: Data-Free Optimal Scaling and
// Pre-Normalization Quantization for MXFP4 Attention") measures its MXFP4
// attention against NVFP4-based baselines.  NVFP4 here is NVIDIA's format:
// E2M1 elements in blocks of 16 with one unsigned E4M3 scale per block, and a
// second fp32 scale per (batch, head) slice of Q, K or V.  All scale
// arithmetic is fp32 with round to nearest:
//   g  = 448 / max(amax_slice, 2^-100)          second-level scale
//   sb = E4M3(amax_block * g)                    round to nearest even, saturating at 448
//   r  = (6 g) / sb   (0 when sb decodes to 0)   element factor
//   code = E2M1(x * r)                           round to nearest even, saturating at 6
// so that value = code * sb / (6 g).
//
//  * nv_amax_kernel: |x| maximum per (tensor, head), an integer max over
//    |bf16| bit patterns folded into the output with atomicMax (the output
//    must be zero first).
//  * nv_quantize_rows_grouped_kernel: Q and K for the attention workspace.  A
//    pair of lanes owns a 16-element block (8 elements each, one 16-byte
//    load); scales go out regrouped per 128 rows and per 64 columns, in the
//    order tcgen05 reads block-16 scale factors (row m, block b of a 64-column
//    chunk at (m % 32) * 16 + (m / 32) * 4 + b of that chunk's 512 bytes).
//  * nv_quantize_vt_kernel: V^T, blocks of 16 tokens per channel, the same
//    regrouping with channels as rows.
//  * nv_quantize_rows_kernel: the standalone op, row-major scales.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

namespace {

constexpr int kNvThreads = 256;

// g = 448 / max(amax, 2^-100), from the fp32 bit pattern of amax.
__device__ __forceinline__ float nv_global(uint32_t amax_bits) {
    return __fdiv_rn(448.f, fmaxf(__uint_as_float(amax_bits), 0x1p-100f));
}

// One 16-element block spread over a pair of lanes (8 elements each): returns
// this lane's 8 packed codes and the block's E4M3 scale byte.
__device__ __forceinline__ uint32_t nv_quantize_pair(uint4 raw, float g, float G, uint32_t& sb_out) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        amax = max(amax, w[i] & 0x7FFFu);
        amax = max(amax, (w[i] >> 16) & 0x7FFFu);
    }
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    const uint32_t sb = e4m3_encode_sat(__fmul_rn(__uint_as_float(amax << 16), g));
    const float sbv = e4m3_decode(sb);
    const float r = sbv > 0.f ? __fdiv_rn(G, sbv) : 0.f;
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), r);
        f[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), r);
    }
    sb_out = sb;
    return pack_e2m1x8(f);
}

__global__ void __launch_bounds__(kNvThreads) nv_amax_kernel(const uint16_t* __restrict__ q,
                                                             const uint16_t* __restrict__ k,
                                                             const uint16_t* __restrict__ v, int64_t per_slice,
                                                             int64_t slices, uint32_t* __restrict__ amax) {
    const uint16_t* x = (blockIdx.z == 0 ? q : (blockIdx.z == 1 ? k : v)) + blockIdx.y * per_slice;
    const int64_t n16 = per_slice / 8;
    uint32_t m = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kNvThreads + threadIdx.x; i < n16;
         i += static_cast<int64_t>(gridDim.x) * kNvThreads) {
        const uint4 r = reinterpret_cast<const uint4*>(x)[i];
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ uint32_t red[kNvThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kNvThreads / 32; ++i) m = max(m, red[i]);
        atomicMax(amax + blockIdx.z * slices + blockIdx.y, m << 16);  // fp32 bits of the bf16 maximum
    }
}

struct NvRowsArgs {
    const uint16_t* x[2];
    uint8_t* codes[2];
    uint8_t* scales[2];
    const uint32_t* amax[2];  // per-slice |x| maxima (fp32 bits)
    float* gs[2];             // per-slice g, written by the first CTA of each slice (may be null)
};

// Q/K for the attention workspace: one CTA per (128-row group, bh, tensor).
template <int D>
__global__ void __launch_bounds__(kNvThreads) nv_quantize_rows_grouped_kernel(NvRowsArgs a, int N, int groups,
                                                                              uint32_t* status) {
    constexpr int kChunksPerRow = D / 8;
    constexpr int kPerThread = 128 * kChunksPerRow / kNvThreads;
    constexpr int kSfBytes = (D / 64) * 512;
    __shared__ __align__(16) uint8_t sf[kSfBytes];
    const bool t1 = blockIdx.z != 0;  // selects, not a dynamic index, keep the arguments in registers
    const uint16_t* __restrict__ x = t1 ? a.x[1] : a.x[0];
    uint32_t* __restrict__ codes = reinterpret_cast<uint32_t*>(t1 ? a.codes[1] : a.codes[0]);
    uint8_t* __restrict__ scales = t1 ? a.scales[1] : a.scales[0];
    float* gs = t1 ? a.gs[1] : a.gs[0];
    const int g = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const float gsc = nv_global((t1 ? a.amax[1] : a.amax[0])[bh]);
    const float G = __fmul_rn(6.f, gsc);
    if (status != nullptr && g == 0 && bh == 0 && !t1 && threadIdx.x == 0) *status = 0u;
    if (g == 0 && threadIdx.x == 0 && gs != nullptr) gs[bh] = gsc;
    for (int i = threadIdx.x; i < kSfBytes / 4; i += kNvThreads) reinterpret_cast<uint32_t*>(sf)[i] = 0u;
    const int64_t row0 = bh * N + static_cast<int64_t>(g) * 128;
    const int rows_valid = min(128, N - g * 128);
    uint4 raw[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int c = threadIdx.x + u * kNvThreads;
        const int m = c / kChunksPerRow;
        raw[u] = (m < rows_valid) ? __ldcs(reinterpret_cast<const uint4*>(x + (row0 + m) * D) + (c % kChunksPerRow))
                                  : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();  // sf cleared
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int c = threadIdx.x + u * kNvThreads;
        const int m = c / kChunksPerRow;
        uint32_t sb;
        const uint32_t packed = nv_quantize_pair(raw[u], gsc, G, sb);
        if (m < rows_valid) codes[(row0 + m) * (D / 8) + (c % kChunksPerRow)] = packed;
        if ((threadIdx.x & 1) == 0) {
            const int j = (c % kChunksPerRow) / 2;  // 16-element block of the row
            sf[(j / 4) * 512 + (m & 31) * 16 + (m >> 5) * 4 + (j % 4)] = static_cast<uint8_t>(sb);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kSfBytes / 16; i += kNvThreads)
        reinterpret_cast<uint4*>(scales + (bh * groups + g) * kSfBytes)[i] = reinterpret_cast<const uint4*>(sf)[i];
}

// V^T: grid (128-token groups, BH), D threads; the CTA stages 128 tokens x D
// channels in shared memory, thread `ch` quantizes the eight 16-token blocks of
// its channel and writes 64 contiguous code bytes and two regrouped scale words.
template <int D>
__global__ void __launch_bounds__(D) nv_quantize_vt_kernel(const uint16_t* __restrict__ v, int N, int npad,
                                                           int groups, const uint32_t* __restrict__ amax,
                                                           float* __restrict__ gs, uint8_t* __restrict__ codes_t,
                                                           uint8_t* __restrict__ scales_t) {
    __shared__ __align__(16) uint16_t tile[128 * D];
    const int g = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int t0 = g * 128;
    const int ch = threadIdx.x;
    const float gsc = nv_global(amax[bh]);
    const float G = __fmul_rn(6.f, gsc);
    if (g == 0 && ch == 0 && gs != nullptr) gs[bh] = gsc;
    constexpr int kChunksPerRow = D / 8;
    constexpr int kPerThread = 128 * kChunksPerRow / D;
    uint4 val[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int c = ch + u * D;
        const int tk = c / kChunksPerRow;
        val[u] = (t0 + tk < N) ? __ldcs(reinterpret_cast<const uint4*>(v + (bh * N + t0 + tk) * D) + (c % kChunksPerRow))
                               : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) reinterpret_cast<uint4*>(tile)[ch + u * D] = val[u];
    __syncthreads();
    uint8_t* rowp = codes_t + (bh * D + ch) * static_cast<int64_t>(npad / 2);
    uint32_t sfw[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint32_t raw[16];
        uint32_t am = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            raw[i] = tile[(16 * k + i) * D + ch];
            am = max(am, raw[i] & 0x7FFFu);
        }
        const uint32_t sb = e4m3_encode_sat(__fmul_rn(__uint_as_float(am << 16), gsc));
        const float sbv = e4m3_decode(sb);
        const float r = sbv > 0.f ? __fdiv_rn(G, sbv) : 0.f;
        uint32_t words[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __fmul_rn(__uint_as_float(raw[8 * w + i] << 16), r);
            words[w] = pack_e2m1x8(f);
        }
        const int tb = t0 + 16 * k;
        if (tb < npad) *reinterpret_cast<uint2*>(rowp + tb / 2) = make_uint2(words[0], words[1]);
        sfw[k / 4] |= sb << (8 * (k % 4));
    }
    uint8_t* grp = scales_t + (bh * groups + g) * 1024;
#pragma unroll
    for (int kc = 0; kc < 2; ++kc) {
        *reinterpret_cast<uint32_t*>(grp + kc * 512 + (ch & 31) * 16 + (ch >> 5) * 4) = sfw[kc];
        if (D < 128) {
            // channel rows D..127 of the atom: scale 1.0 (E4M3 0x38), so the ones-row the
            // attention kernel appends to V^T (row D) is read with unit scale
            const int c2 = ch + D;
            *reinterpret_cast<uint32_t*>(grp + kc * 512 + (c2 & 31) * 16 + (c2 >> 5) * 4) = 0x38383838u;
        }
    }
}

// Standalone op: rows of `cols` elements, row-major scales [rows, cols/16];
// grid-stride over 16-byte chunks.  The second-level scale comes from gs[0]
// (the tensor's amax, fp32 bits); the first CTA writes g to gs[1].
__global__ void __launch_bounds__(kNvThreads) nv_quantize_rows_kernel(const uint16_t* __restrict__ x, int64_t n_chunks,
                                                                      uint8_t* __restrict__ codes_b,
                                                                      uint8_t* __restrict__ scales, float* gs) {
    uint32_t* __restrict__ codes = reinterpret_cast<uint32_t*>(codes_b);
    const float gsc = nv_global(__float_as_uint(gs[0]));
    const float G = __fmul_rn(6.f, gsc);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kNvThreads;
    // every lane of a warp takes part in the pair shuffle: the loop runs per warp
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * kNvThreads + (threadIdx.x - lane);
    for (int64_t base = warp0; base < n_chunks; base += stride) {
        const int64_t i = base + lane;
        const uint4 raw = (i < n_chunks) ? __ldcs(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0, 0, 0, 0);
        uint32_t sb;
        const uint32_t packed = nv_quantize_pair(raw, gsc, G, sb);
        if (i < n_chunks) {
            codes[i] = packed;
            if ((i & 1) == 0) scales[i >> 1] = static_cast<uint8_t>(sb);
        }
    }
}

__global__ void nv_store_global_kernel(float* gs) {
    // gs[1] = g of the amax in gs[0] (one thread; after the quantizer read gs[0])
    gs[1] = nv_global(__float_as_uint(gs[0]));
}

int nv_grid(int64_t work_items, int per_block, int ctas_per_sm) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (work_items + per_block - 1) / per_block;
    const int64_t cap = static_cast<int64_t>(sms) * ctas_per_sm;
    return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_nv_amax(const void* q, const void* k, const void* v, int ntensors, int64_t per_slice,
                           int64_t slices, uint32_t* amax, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(uint32_t) * ntensors * slices, stream);
    if (e != cudaSuccess) return e;
    // about 8 CTAs per SM in all, split over the slices
    const int64_t total = nv_grid(per_slice / 8 * slices * ntensors, kNvThreads, 8);
    int64_t per = total / (slices * ntensors);
    if (per < 1) per = 1;
    const int64_t need = (per_slice / 8 + kNvThreads - 1) / kNvThreads;
    if (per > need) per = need;
    dim3 grid(static_cast<unsigned>(per), static_cast<unsigned>(slices), ntensors);
    nv_amax_kernel<<<grid, kNvThreads, 0, stream>>>(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                                    static_cast<const uint16_t*>(v), per_slice, slices, amax);
    return cudaGetLastError();
}

cudaError_t launch_nv_quantize_qk(const void* q, const void* k, uint8_t* q_codes, uint8_t* k_codes, uint8_t* q_sf,
                                  uint8_t* k_sf, const uint32_t* amax_q, const uint32_t* amax_k, float* gs_q,
                                  float* gs_k, int64_t BH, int N, int d, int groups, uint32_t* status,
                                  cudaStream_t stream) {
    NvRowsArgs a{};
    a.x[0] = static_cast<const uint16_t*>(q);
    a.x[1] = static_cast<const uint16_t*>(k);
    a.codes[0] = q_codes;
    a.codes[1] = k_codes;
    a.scales[0] = q_sf;
    a.scales[1] = k_sf;
    a.amax[0] = amax_q;
    a.amax[1] = amax_k;
    a.gs[0] = gs_q;
    a.gs[1] = gs_k;
    dim3 grid(groups, static_cast<unsigned>(BH), 2);
    if (d == 128)
        nv_quantize_rows_grouped_kernel<128><<<grid, kNvThreads, 0, stream>>>(a, N, groups, status);
    else
        nv_quantize_rows_grouped_kernel<64><<<grid, kNvThreads, 0, stream>>>(a, N, groups, status);
    return cudaGetLastError();
}

cudaError_t launch_nv_quantize_vt(const void* v, int64_t BH, int N, int d, int groups, const uint32_t* amax_v,
                                  float* gs_v, uint8_t* codes_t, uint8_t* scales_t, cudaStream_t stream) {
    const int npad = (N + 31) / 32 * 32;
    dim3 grid(groups, static_cast<unsigned>(BH));
    if (d == 128)
        nv_quantize_vt_kernel<128><<<grid, 128, 0, stream>>>(static_cast<const uint16_t*>(v), N, npad, groups, amax_v,
                                                              gs_v, codes_t, scales_t);
    else
        nv_quantize_vt_kernel<64><<<grid, 64, 0, stream>>>(static_cast<const uint16_t*>(v), N, npad, groups, amax_v,
                                                            gs_v, codes_t, scales_t);
    return cudaGetLastError();
}

cudaError_t launch_nv_quantize_rows(const void* x, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                                    float* gs, cudaStream_t stream) {
    const int64_t n = rows * cols;
    cudaError_t e = launch_nv_amax(x, x, x, 1, n, 1, reinterpret_cast<uint32_t*>(gs), stream);
    if (e != cudaSuccess) return e;
    const int64_t n_chunks = n / 8;
    nv_quantize_rows_kernel<<<nv_grid(n_chunks, kNvThreads, 8), kNvThreads, 0, stream>>>(
        static_cast<const uint16_t*>(x), n_chunks, codes, scales, gs);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    nv_store_global_kernel<<<1, 1, 0, stream>>>(gs);
    return cudaGetLastError();
}

}  // namespace mxattn
