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

// MXFP4 quantization of one 32-element bf16 block spread over a quad of lanes
// (lanes 4k .. 4k + 3, 8 elements each in `raw`): the block maximum is an
// integer max over |bf16| bit patterns plus two xor shuffles, e its block
// exponent under the scale boundary `mant_thresh`; returns this lane's 8 E2M1
// codes packed (element 0 in the lowest nibble).  All 32 lanes must call it.
__device__ __forceinline__ uint32_t quantize_quad_bf16(uint4 raw, uint32_t mant_thresh, int& e_out) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        amax = max(amax, w[i] & 0x7FFFu);
        amax = max(amax, (w[i] >> 16) & 0x7FFFu);
    }
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = block_exponent_bf16(amax, mant_thresh);
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

// MXFP4 quantization of two channels over one 32-token block of V: raw[i] holds
// token i's channel 2c in its low half and channel 2c + 1 in its high half.
// words[h][0..3] get channel 2c + h's 32 codes (token 0 in the lowest nibble of
// words[h][0]), e[h] its block exponent.
__device__ __forceinline__ void quantize_vt_block_bf16(const uint32_t (&raw)[32], uint32_t mant_thresh,
                                                       uint32_t (&words)[2][4], int (&e)[2]) {
    uint32_t amax0 = 0, amax1 = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        amax0 = max(amax0, raw[i] & 0x7FFFu);
        amax1 = max(amax1, (raw[i] >> 16) & 0x7FFFu);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        e[h] = block_exponent_bf16(h ? amax1 : amax0, mant_thresh);
        const float sc = exp2_neg_int(e[h]);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                f[i] = __uint_as_float(h ? (raw[8 * w + i] & 0xFFFF0000u) : (raw[8 * w + i] << 16)) * sc;
            words[h][w] = pack_e2m1x8(f);
        }
    }
}

}  // namespace mxattn
