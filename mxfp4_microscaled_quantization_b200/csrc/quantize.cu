// quantize.cu -- HBM-bound MXFP4 quantize/pack kernels for sm_100a.
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
// Quantization for MXFP4 Attention", abstract -- MXFP4 operands with
// power-of-two microscaling; scale rule OCP (floor(log2 amax) - 2) or UOS
// (smallest e with amax <= Qmax * 2^e, Qmax = 7.25).
//
//  * quantize_rows_kernel: blocks of 32 consecutive elements of a row (Q, K,
//    and the standalone op).  Each thread loads 16 bytes (8 bf16), a quad of
//    lanes owns one block: the block maximum is an integer max over |bf16|
//    bit patterns plus two xor-shuffles, the exponent comes from the maximum's
//    exponent and mantissa fields, the 8 scaled values go through four
//    cvt.rn.satfinite.e2m1x2 and leave as one 32-bit store.  The quad's first
//    lane stores the E8M0 byte (row-major, or regrouped per 128 rows in the
//    order the tensor core reads scale factors).
//  * quantize_vt_kernel: V blocks of 32 consecutive tokens per channel,
//    written transposed (V^T, tokens contiguous): a CTA stages 128 tokens x d
//    channels in shared memory and each thread quantizes (channel, block)
//    columns from there.
//  * regroup_sf_kernel: row-major scales -> the 128-row regrouped order.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mxattn {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kUnroll = 4;

// One 32-element block spread over a quad of lanes (8 elements each).
// Returns the packed codes of this lane's 8 elements; `e_out` gets the block exponent.
__device__ __forceinline__ uint32_t quantize_quad(uint4 raw, int uos, int& e_out) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        amax = max(amax, w[i] & 0x7FFFu);
        amax = max(amax, (w[i] >> 16) & 0x7FFFu);
    }
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = block_exponent_bf16(amax, uos);
    const float sc = exp2_neg_int(e);
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16) * sc;
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u) * sc;
    }
    e_out = e;
    return pack_e2m1x8(f);
}

// Regrouped scale offset of (row r of a [*, N] operand, block k): per 128-row
// group, row m sits at byte (m%32)*16 + (m/32)*4 + k.
__device__ __forceinline__ int64_t regrouped_sf_offset(int64_t bh, int64_t groups, int r, int k) {
    const int m = r & 127;
    return (bh * groups + (r >> 7)) * 512 + (m & 31) * 16 + (m >> 5) * 4 + k;
}

struct RowsArgs {
    const uint16_t* x[2];
    uint8_t* codes[2];
    uint8_t* scales[2];
};

// Row quantization of up to two tensors (blockIdx.y selects one).
//   n_chunks: 16-byte chunks per tensor (rows * cols / 8).
//   regroup == 0: scales are row-major [rows, cols/32].
//   regroup == 1: rows are (bh, r) with r < N; scales go to the regrouped
//     layout (cols in {64, 128}) and the scale bytes of the padding rows
//     r in [N, G*128) are zeroed.
__global__ void __launch_bounds__(kQuantThreads) quantize_rows_kernel(RowsArgs a, int64_t n_chunks, int cols,
                                                                      int uos, int regroup, int N, int groups,
                                                                      int64_t BH, uint32_t* status) {
    const uint16_t* __restrict__ x = a.x[blockIdx.y];
    uint32_t* __restrict__ codes = reinterpret_cast<uint32_t*>(a.codes[blockIdx.y]);
    uint8_t* __restrict__ scales = a.scales[blockIdx.y];
    if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status = 0u;

    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
    const int chunk_shift = (cols == 64) ? 3 : 4;  // log2(chunks per row) in regrouped mode
    const int blocks_per_row = cols >> 5;

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
            const uint32_t packed = quantize_quad(raw[u], uos, e);
            if (i < n_chunks) {
                codes[i] = packed;
                if ((lane & 3) == 0) {
                    const int64_t blk = i >> 2;
                    if (!regroup) {
                        scales[blk] = static_cast<uint8_t>(e + 127);
                    } else {
                        const int64_t row = i >> chunk_shift;
                        const int k = static_cast<int>(blk % blocks_per_row);
                        const int64_t bh = row / N;
                        const int r = static_cast<int>(row - bh * N);
                        scales[regrouped_sf_offset(bh, groups, r, k)] = static_cast<uint8_t>(e + 127);
                    }
                }
            }
        }
    }
    if (regroup) {
        // zero the scale bytes of padding rows so the tensor core never reads stale bytes
        const int pad_rows = groups * 128 - N;
        const int64_t n_pad = BH * pad_rows * blocks_per_row;
        const int64_t tid = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x;
        for (int64_t t = tid; t < n_pad; t += static_cast<int64_t>(gridDim.x) * kQuantThreads) {
            const int k = static_cast<int>(t % blocks_per_row);
            const int64_t pr = t / blocks_per_row;
            const int64_t bh = pr / pad_rows;
            const int r = N + static_cast<int>(pr - bh * pad_rows);
            scales[regrouped_sf_offset(bh, groups, r, k)] = 0;
        }
    }
}

// V^T quantization: grid (G token groups of 128, BH).  Shared tile [128][D] bf16.
template <int D>
__global__ void __launch_bounds__(kQuantThreads) quantize_vt_kernel(const uint16_t* __restrict__ v, int N, int npad,
                                                                    int uos, int regroup, int groups,
                                                                    uint8_t* __restrict__ codes_t,
                                                                    uint8_t* __restrict__ scales_t) {
    __shared__ __align__(16) uint16_t tile[128 * D];
    const int g = blockIdx.x;
    const int64_t bh = blockIdx.y;
    const int t0 = g * 128;
    constexpr int kChunksPerRow = D / 8;
    for (int c = threadIdx.x; c < 128 * kChunksPerRow; c += kQuantThreads) {
        const int t = c / kChunksPerRow, q = c % kChunksPerRow;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (t0 + t < N) val = __ldcs(reinterpret_cast<const uint4*>(v + ((bh * N + t0 + t) * D)) + q);
        reinterpret_cast<uint4*>(tile)[c] = val;
    }
    __syncthreads();
    for (int item = threadIdx.x; item < D * 4; item += kQuantThreads) {
        const int ch = item % D, k = item / D;
        uint32_t amax = 0;
        uint32_t raw[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            raw[i] = tile[(32 * k + i) * D + ch];
            amax = max(amax, raw[i] & 0x7FFFu);
        }
        const int e = block_exponent_bf16(amax, uos);
        const float sc = exp2_neg_int(e);
        uint32_t words[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(raw[8 * w + i] << 16) * sc;
            words[w] = pack_e2m1x8(f);
        }
        const int tb = t0 + 32 * k;  // first token of the block
        if (tb < npad) {
            uint8_t* dst = codes_t + (bh * D + ch) * static_cast<int64_t>(npad / 2) + tb / 2;
            *reinterpret_cast<uint4*>(dst) = make_uint4(words[0], words[1], words[2], words[3]);
        }
        const uint8_t sbyte = static_cast<uint8_t>(e + 127);
        if (!regroup) {
            if (tb < npad) scales_t[(bh * D + ch) * static_cast<int64_t>(npad / 32) + tb / 32] = sbyte;
        } else {
            // group g of 128 tokens; channel ch plays the role of the row
            scales_t[(bh * groups + g) * 512 + (ch & 31) * 16 + (ch >> 5) * 4 + k] = sbyte;
        }
    }
    if (regroup && D < 128) {
        // channel rows D..127 of the group: scale 2^0, so the extra ones-row the
        // attention kernel appends to V^T (row D) is read with unit scale
        for (int idx = threadIdx.x; idx < (128 - D) * 4; idx += kQuantThreads) {
            const int ch = D + idx / 4, k = idx % 4;
            scales_t[(bh * groups + g) * 512 + (ch & 31) * 16 + (ch >> 5) * 4 + k] = 127;
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
    const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 resident CTAs of 256 threads per SM
    return static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_quantize_rows(const void* const* x, uint8_t* const* codes, uint8_t* const* scales, int ntensors,
                                 int64_t rows, int cols, int uos, int regroup, int N, int groups, int64_t BH,
                                 uint32_t* status, cudaStream_t stream) {
    RowsArgs a{};
    for (int t = 0; t < ntensors; ++t) {
        a.x[t] = static_cast<const uint16_t*>(x[t]);
        a.codes[t] = codes[t];
        a.scales[t] = scales[t];
    }
    const int64_t n_chunks = rows * cols / 8;
    dim3 grid(grid_for(n_chunks / kUnroll, kQuantThreads), ntensors);
    quantize_rows_kernel<<<grid, kQuantThreads, 0, stream>>>(a, n_chunks, cols, uos, regroup, N, groups, BH, status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_vt(const void* v, int64_t BH, int N, int d, int uos, int regroup, int groups,
                               uint8_t* codes_t, uint8_t* scales_t, cudaStream_t stream) {
    const int npad = (N + 31) / 32 * 32;
    dim3 grid(groups, static_cast<unsigned>(BH));
    if (d == 128)
        quantize_vt_kernel<128><<<grid, kQuantThreads, 0, stream>>>(static_cast<const uint16_t*>(v), N, npad, uos,
                                                                    regroup, groups, codes_t, scales_t);
    else
        quantize_vt_kernel<64><<<grid, kQuantThreads, 0, stream>>>(static_cast<const uint16_t*>(v), N, npad, uos,
                                                                   regroup, groups, codes_t, scales_t);
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
