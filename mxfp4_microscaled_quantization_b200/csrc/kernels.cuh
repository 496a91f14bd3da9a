// kernels.cuh -- host-side launchers shared by the C-ABI entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "mxattn.h"

namespace mxattn {

// Largest sequence length the attention entry points accept.
constexpr int64_t kMaxAttentionN = int64_t(1) << 24;

// The argument checks every attention entry point runs first, in this order:
// B, H, N >= 1 and O non-null (else MXATTN_ERR_INVALID), pnq in {0, 1}
// (INVALID), d in {64, 128} and kv_tile in {64, 128} (MXATTN_ERR_UNSUPPORTED),
// N <= kMaxAttentionN and the grid size (UNSUPPORTED).
mxattn_status check_attention_shape(int B, int H, int N, int d, int kv_tile, int pnq, const float* O);

// Row quantization of a bf16 tensor [rows, cols] (cols a multiple of 32) with
// row-major scales [rows, cols/32].  Clears *status when status != nullptr.
cudaError_t launch_quantize_rows(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows, int cols,
                                 uint32_t sf_thresh, uint32_t* status, cudaStream_t stream);

// V [BH, N, d] -> V^T codes [BH, d, Npad/2] and row-major scales [BH, d, Npad/32].
cudaError_t launch_quantize_vt(const void* v, int64_t BH, int N, int d, uint32_t sf_thresh, uint8_t* codes_t,
                               uint8_t* scales_t, cudaStream_t stream);

// The forward's operand preparation in one persistent launch: Q and K [BH, N,
// d] bf16 -> codes [BH, N, d/2] + regrouped scales, V -> V^T codes [BH, d,
// Npad/2] + regrouped scales (channel rows d..127 of each group at scale 2^0).
// Clears *status.  Q, K, V 16-byte aligned.
cudaError_t launch_prepare(const void* Q, const void* K, const void* V, int64_t BH, int N, int d, uint32_t sf_thresh,
                           int groups, uint8_t* q_codes, uint8_t* k_codes, uint8_t* vt_codes, uint8_t* q_sf,
                           uint8_t* k_sf, uint8_t* v_sf, uint32_t* status, cudaStream_t stream);

// cuTensorMapEncodeTiled through the runtime's driver entry point (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Row-major Q/K/V^T scales -> regrouped scales; clears *status.
cudaError_t launch_regroup_sf(const uint8_t* q_scales, const uint8_t* k_scales, const uint8_t* vt_scales, int64_t BH,
                              int N, int d, int groups, uint8_t* q_sf, uint8_t* k_sf, uint8_t* v_sf,
                              uint32_t* status, cudaStream_t stream);

struct AttnArgs {
    const uint8_t* q_codes;  // [BH, N, d/2]
    const uint8_t* k_codes;  // [BH, N, d/2]
    const uint8_t* vt_codes; // [BH, d, Npad/2]
    const uint8_t* q_sf;     // regrouped, [BH, G, 512] (NVFP4: [BH, G, (d/64)*512]; V^T [BH, G, 1024])
    const uint8_t* k_sf;
    const uint8_t* v_sf;
    float* O;                // [BH, N, d]
    uint32_t* status;
    int64_t BH;
    int N;
    int d;
    int kv_tile;
    int pnq;
    float qmax;         // scale boundary of P's block exponents, in (4, 8] (8 = OCP)
    float softmax_scale;
    int nv;             // 1: NVFP4 operands (16-element blocks, E4M3 scales) instead of MXFP4
    const float* gs;    // NVFP4: second-level scales g of Q, K, V per (b, h), [3][BH]
};

// NVFP4 (comparison variant).  Per-slice |x| maxima of ntensors (1..3)
// tensors of `slices` slices of per_slice elements each, as fp32 bit
// patterns, into amax[ntensors * slices] (zeroed first).
cudaError_t launch_nv_amax(const void* q, const void* k, const void* v, int ntensors, int64_t per_slice,
                           int64_t slices, uint32_t* amax, cudaStream_t stream);
// Q and K [BH, N, d] -> codes [BH, N, d/2] + regrouped E4M3 scales [BH, G, (d/64)*512];
// g per slice into gs_q / gs_k (may be null); clears *status.
cudaError_t launch_nv_quantize_qk(const void* q, const void* k, uint8_t* q_codes, uint8_t* k_codes, uint8_t* q_sf,
                                  uint8_t* k_sf, const uint32_t* amax_q, const uint32_t* amax_k, float* gs_q,
                                  float* gs_k, int64_t BH, int N, int d, int groups, uint32_t* status,
                                  cudaStream_t stream);
// V [BH, N, d] -> V^T codes [BH, d, Npad/2] + regrouped E4M3 scales [BH, G, 1024]; g into gs_v.
cudaError_t launch_nv_quantize_vt(const void* v, int64_t BH, int N, int d, int groups, const uint32_t* amax_v,
                                  float* gs_v, uint8_t* codes_t, uint8_t* scales_t, cudaStream_t stream);
// Standalone: x [rows, cols] -> codes [rows, cols/2] + row-major E4M3 scales [rows, cols/16];
// gs (device, 2 floats) receives the amax and g.
cudaError_t launch_nv_quantize_rows(const void* x, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                                    float* gs, cudaStream_t stream);

// The fused attention kernel.  Returns cudaSuccess or the launch / encode error.
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t stream);

}  // namespace mxattn
