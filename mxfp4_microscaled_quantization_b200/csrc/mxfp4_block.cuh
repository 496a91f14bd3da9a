// mxfp4_block.cuh -- MXFP4 quantization of 32-element bf16 blocks, shared by the
// forward's fused preparation (prepare.cu) and the standalone quantizers
// (quantize.cu).
//
// Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
// Quantization for MXFP4 Attention", abstract -- MXFP4 with power-of-two
// microscaling: per block of 32 elements the exponent e from the block's
// largest magnitude (scale rule OCP or UOS, as a mantissa threshold on the
// bf16 maximum), then each element / 2^e rounded to E2M1.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace mxattn {

// Lane-wise maximum of two pairs of unsigned 16-bit values.
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// The block maximum works on |bf16| bit patterns (sign cleared), which order
// like the magnitudes, two per 32-bit word at a time; the scaling multiplies
// two fp32 values per instruction by the power of two 2^-e (exact, round to
// nearest even like the scalar product).

// MXFP4 quantization of one 32-element bf16 block spread over a quad of lanes
// (lanes 4k .. 4k + 3, 8 elements each in `raw`): the block maximum is a
// maximum over |bf16| bit patterns plus two xor shuffles, e its block exponent
// under the scale boundary `mant_thresh`; returns this lane's 8 E2M1 codes
// packed (element 0 in the lowest nibble).  All 32 lanes must call it.
__device__ __forceinline__ uint32_t quantize_quad_bf16(uint4 raw, uint32_t mant_thresh, int& e_out) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    const uint32_t m2 = vmax_u16x2(vmax_u16x2(w[0] & 0x7FFF7FFFu, w[1] & 0x7FFF7FFFu),
                                   vmax_u16x2(w[2] & 0x7FFF7FFFu, w[3] & 0x7FFF7FFFu));
    uint32_t amax = max(m2 & 0xFFFFu, m2 >> 16);
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = block_exponent_bf16(amax, mant_thresh);
    const float sc = exp2_neg_int(e);
    uint32_t f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) fmul2_bcast(f[2 * i], f[2 * i + 1], w[i] << 16, w[i] & 0xFFFF0000u, sc);
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(f[i]);
    e_out = e;
    return pack_e2m1x8(v);
}

// MXFP4 quantization of two channels over one 32-token block of V: raw[i] holds
// token i's channel 2c in its low half and channel 2c + 1 in its high half.
// words[h][0..3] get channel 2c + h's 32 codes (token 0 in the lowest nibble of
// words[h][0]), e[h] its block exponent.
__device__ __forceinline__ void quantize_vt_block_bf16(const uint32_t (&raw)[32], uint32_t mant_thresh,
                                                       uint32_t (&words)[2][4], int (&e)[2]) {
    uint32_t m2 = raw[0] & 0x7FFF7FFFu;
#pragma unroll
    for (int i = 1; i < 32; ++i) m2 = vmax_u16x2(m2, raw[i] & 0x7FFF7FFFu);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        e[h] = block_exponent_bf16(h ? (m2 >> 16) : (m2 & 0xFFFFu), mant_thresh);
        const float sc = exp2_neg_int(e[h]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t f[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const uint32_t a = raw[8 * w + i], b = raw[8 * w + i + 1];
                fmul2_bcast(f[i], f[i + 1], h ? (a & 0xFFFF0000u) : (a << 16), h ? (b & 0xFFFF0000u) : (b << 16), sc);
            }
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(f[i]);
            words[h][w] = pack_e2m1x8(v);
        }
    }
}

}  // namespace mxattn
