// api.cu -- the C ABI of libmxattn.so (declared in include/mxattn.h):
// argument checks, workspace layout, kernel launches.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.cuh"
#include "mxattn.h"

#define MXATTN_API extern "C" __attribute__((visibility("default")))

namespace mxattn {

mxattn_status check_attention_shape(int B, int H, int N, int d, int kv_tile, int pnq, const float* O) {
    if (B < 1 || H < 1 || N < 1 || O == nullptr) return MXATTN_ERR_INVALID;
    if (pnq != 0 && pnq != 1) return MXATTN_ERR_INVALID;
    if (d != 64 && d != 128) return MXATTN_ERR_UNSUPPORTED;
    if (kv_tile != 64 && kv_tile != 128) return MXATTN_ERR_UNSUPPORTED;
    if (N > kMaxAttentionN || static_cast<int64_t>(B) * H > (int64_t(1) << 31) / ((N + 127) / 128))
        return MXATTN_ERR_UNSUPPORTED;
    return MXATTN_OK;
}

}  // namespace mxattn

namespace {

constexpr int64_t kMaxN = mxattn::kMaxAttentionN;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
    size_t status, q_codes, k_codes, vt_codes, q_sf, k_sf, v_sf, total;
};

bool make_layout(int B, int H, int N, int d, Layout* L) {
    if (B < 1 || H < 1 || N < 1 || N > kMaxN || (d != 64 && d != 128)) return false;
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t G = (static_cast<size_t>(N) + 127) / 128;
    const size_t npad = (static_cast<size_t>(N) + 31) / 32 * 32;
    size_t off = 0;
    L->status = off;
    off += 256;
    L->q_codes = off;
    off = align256(off + BH * N * d / 2);
    L->k_codes = off;
    off = align256(off + BH * N * d / 2);
    L->vt_codes = off;
    off = align256(off + BH * d * npad / 2);
    L->q_sf = off;
    off = align256(off + BH * G * 512);
    L->k_sf = off;
    off = align256(off + BH * G * 512);
    L->v_sf = off;
    off = align256(off + BH * G * 512);
    L->total = off;
    return true;
}

// Mantissa thresholds of the block-exponent rule for a scale boundary Qmax in
// (4, 8]: the smallest e with amax <= Qmax * 2^e is floor(log2 amax) - 2 plus
// one when amax's significand exceeds Qmax / 4.  Qmax = 8 is the OCP rule
// e = floor(log2 amax) - 2 (the significand never exceeds 2).
struct Thresholds {
    uint32_t bf16;  // 7-bit mantissa field
};

bool qmax_thresholds(float qmax, Thresholds* t) {
    if (!(qmax > 4.f && qmax <= 8.f)) return false;  // also rejects NaN
    const double r = static_cast<double>(qmax) / 4.0 - 1.0;  // in (0, 1]
    t->bf16 = qmax == 8.f ? 0x7Fu : static_cast<uint32_t>(std::floor(r * 128.0));
    return true;
}

// The boundary a named rule stands for: OCP = 8, UOS = 7.25 (the abstract's Qmax).
bool rule_qmax(mxattn_rule rule, float* qmax) {
    if (rule == MXATTN_RULE_OCP) *qmax = 8.f;
    else if (rule == MXATTN_RULE_UOS) *qmax = 7.25f;
    else return false;
    return true;
}

mxattn_status check_attention_args(int B, int H, int N, int d, int kv_tile, int pnq, const float* O, const void* ws,
                                   size_t ws_bytes, Layout* L) {
    if (ws == nullptr) return MXATTN_ERR_INVALID;
    const mxattn_status st = mxattn::check_attention_shape(B, H, N, d, kv_tile, pnq, O);
    if (st != MXATTN_OK) return st;
    if (!make_layout(B, H, N, d, L)) return MXATTN_ERR_INVALID;
    if (ws_bytes < L->total || !aligned(ws, 256) || !aligned(O, 16)) return MXATTN_ERR_INVALID;
    return MXATTN_OK;
}

float resolve_scale(float s, int d) { return (s > 0.f) ? s : static_cast<float>(1.0 / std::sqrt(static_cast<double>(d))); }

}  // namespace

MXATTN_API const char* mxattn_status_string(mxattn_status status) {
    switch (status) {
        case MXATTN_OK: return "ok";
        case MXATTN_ERR_INVALID: return "invalid argument";
        case MXATTN_ERR_UNSUPPORTED: return "unsupported shape or tile";
        case MXATTN_ERR_CUDA: return "CUDA error";
        case MXATTN_ERR_TIMEOUT: return "a bounded wait in the attention kernel timed out";
    }
    return "unknown status";
}

MXATTN_API mxattn_status mxattn_quantize_qmax(const void* x, int64_t rows, int64_t cols, float qmax, uint8_t* codes,
                                              uint8_t* scales, mxattn_stream_t stream) {
    Thresholds th;
    if (rows < 0 || cols <= 0 || cols % 32 != 0 || !qmax_thresholds(qmax, &th)) return MXATTN_ERR_INVALID;
    if (rows == 0) return MXATTN_OK;
    if (x == nullptr || codes == nullptr || scales == nullptr) return MXATTN_ERR_INVALID;
    if (!aligned(x, 16) || !aligned(codes, 4)) return MXATTN_ERR_INVALID;
    if (rows > (int64_t(1) << 40) / cols) return MXATTN_ERR_UNSUPPORTED;
    cudaError_t e = mxattn::launch_quantize_rows(x, codes, scales, rows, static_cast<int>(cols), th.bf16, nullptr,
                                                 reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_quantize(const void* x, int64_t rows, int64_t cols, mxattn_rule rule, uint8_t* codes,
                                         uint8_t* scales, mxattn_stream_t stream) {
    float q;
    if (!rule_qmax(rule, &q)) return MXATTN_ERR_INVALID;
    return mxattn_quantize_qmax(x, rows, cols, q, codes, scales, stream);
}

MXATTN_API mxattn_status mxattn_quantize_vt(const void* v, int64_t BH, int64_t N, int64_t d, mxattn_rule rule,
                                            uint8_t* codes_t, uint8_t* scales_t, mxattn_stream_t stream) {
    if (v == nullptr || codes_t == nullptr || scales_t == nullptr || BH < 1 || N < 1) return MXATTN_ERR_INVALID;
    float q;
    Thresholds th;
    if (!rule_qmax(rule, &q) || !qmax_thresholds(q, &th)) return MXATTN_ERR_INVALID;
    if (d != 64 && d != 128) return MXATTN_ERR_UNSUPPORTED;
    if (N > kMaxN || BH > 65535) return MXATTN_ERR_UNSUPPORTED;
    if (!aligned(v, 16) || !aligned(codes_t, 16)) return MXATTN_ERR_INVALID;
    cudaError_t e = mxattn::launch_quantize_vt(v, BH, static_cast<int>(N), static_cast<int>(d), th.bf16, codes_t,
                                               scales_t, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API size_t mxattn_workspace_size(int B, int H, int N, int d) {
    Layout L;
    return make_layout(B, H, N, d, &L) ? L.total : 0;
}

MXATTN_API mxattn_status mxattn_prepare_qmax(const void* Q, const void* K, const void* V, int B, int H, int N,
                                             int d, float qmax, void* workspace, size_t workspace_bytes,
                                             mxattn_stream_t stream) {
    Layout L;
    float dummy_out[4];
    Thresholds th;
    if (!qmax_thresholds(qmax, &th)) return MXATTN_ERR_INVALID;
    mxattn_status st = check_attention_args(B, H, N, d, 128, 1, dummy_out, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    if (Q == nullptr || K == nullptr || V == nullptr) return MXATTN_ERR_INVALID;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16)) return MXATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    const int64_t BH = static_cast<int64_t>(B) * H;
    const int G = (N + 127) / 128;
    cudaError_t e = mxattn::launch_prepare(Q, K, V, BH, N, d, th.bf16, G, ws + L.q_codes, ws + L.k_codes,
                                           ws + L.vt_codes, ws + L.q_sf, ws + L.k_sf, ws + L.v_sf, status, s);
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_prepare(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                        mxattn_rule rule, void* workspace, size_t workspace_bytes,
                                        mxattn_stream_t stream) {
    float q;
    if (!rule_qmax(rule, &q)) return MXATTN_ERR_INVALID;
    return mxattn_prepare_qmax(Q, K, V, B, H, N, d, q, workspace, workspace_bytes, stream);
}

MXATTN_API mxattn_status mxattn_attend_qmax(int B, int H, int N, int d, int kv_tile, int pnq, float qmax,
                                            float softmax_scale, float* O, void* workspace, size_t workspace_bytes,
                                            mxattn_stream_t stream) {
    Layout L;
    Thresholds th;
    if (!qmax_thresholds(qmax, &th)) return MXATTN_ERR_INVALID;
    mxattn_status st = check_attention_args(B, H, N, d, kv_tile, pnq, O, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    mxattn::AttnArgs a{};
    a.q_codes = ws + L.q_codes;
    a.k_codes = ws + L.k_codes;
    a.vt_codes = ws + L.vt_codes;
    a.q_sf = ws + L.q_sf;
    a.k_sf = ws + L.k_sf;
    a.v_sf = ws + L.v_sf;
    a.O = O;
    a.status = reinterpret_cast<uint32_t*>(ws + L.status);
    a.BH = static_cast<int64_t>(B) * H;
    a.N = N;
    a.d = d;
    a.kv_tile = kv_tile;
    a.pnq = pnq;
    a.qmax = qmax;
    a.softmax_scale = resolve_scale(softmax_scale, d);
    cudaError_t e = mxattn::launch_attention(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_attend(int B, int H, int N, int d, int kv_tile, int pnq, mxattn_rule rule,
                                       float softmax_scale, float* O, void* workspace, size_t workspace_bytes,
                                       mxattn_stream_t stream) {
    float q;
    if (!rule_qmax(rule, &q)) return MXATTN_ERR_INVALID;
    return mxattn_attend_qmax(B, H, N, d, kv_tile, pnq, q, softmax_scale, O, workspace, workspace_bytes, stream);
}

MXATTN_API mxattn_status mxattn_forward_qmax(const void* Q, const void* K, const void* V, int B, int H, int N,
                                             int d, int kv_tile, int pnq, float qmax, float softmax_scale, float* O,
                                             void* workspace, size_t workspace_bytes, mxattn_stream_t stream) {
    Layout L;
    Thresholds th;
    if (!qmax_thresholds(qmax, &th)) return MXATTN_ERR_INVALID;
    mxattn_status st = check_attention_args(B, H, N, d, kv_tile, pnq, O, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    st = mxattn_prepare_qmax(Q, K, V, B, H, N, d, qmax, workspace, workspace_bytes, stream);
    if (st != MXATTN_OK) return st;
    return mxattn_attend_qmax(B, H, N, d, kv_tile, pnq, qmax, softmax_scale, O, workspace, workspace_bytes, stream);
}

MXATTN_API mxattn_status mxattn_forward(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                        int kv_tile, int pnq, mxattn_rule rule, float softmax_scale, float* O,
                                        void* workspace, size_t workspace_bytes, mxattn_stream_t stream) {
    float q;
    if (!rule_qmax(rule, &q)) return MXATTN_ERR_INVALID;
    return mxattn_forward_qmax(Q, K, V, B, H, N, d, kv_tile, pnq, q, softmax_scale, O, workspace, workspace_bytes,
                               stream);
}

MXATTN_API mxattn_status mxattn_forward_quantized(const uint8_t* q_codes, const uint8_t* q_scales,
                                                  const uint8_t* k_codes, const uint8_t* k_scales,
                                                  const uint8_t* vt_codes, const uint8_t* vt_scales, int B, int H,
                                                  int N, int d, int kv_tile, int pnq, mxattn_rule rule,
                                                  float softmax_scale, float* O, void* workspace,
                                                  size_t workspace_bytes, mxattn_stream_t stream) {
    Layout L;
    float q;
    Thresholds th;
    if (!rule_qmax(rule, &q) || !qmax_thresholds(q, &th)) return MXATTN_ERR_INVALID;
    mxattn_status st = check_attention_args(B, H, N, d, kv_tile, pnq, O, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    if (!q_codes || !q_scales || !k_codes || !k_scales || !vt_codes || !vt_scales) return MXATTN_ERR_INVALID;
    if (!aligned(q_codes, 16) || !aligned(k_codes, 16) || !aligned(vt_codes, 16)) return MXATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
    const int64_t BH = static_cast<int64_t>(B) * H;
    const int G = (N + 127) / 128;
    cudaError_t e = mxattn::launch_regroup_sf(q_scales, k_scales, vt_scales, BH, N, d, G, ws + L.q_sf, ws + L.k_sf,
                                              ws + L.v_sf, status, s);
    if (e != cudaSuccess) return MXATTN_ERR_CUDA;
    mxattn::AttnArgs a{};
    a.q_codes = q_codes;
    a.k_codes = k_codes;
    a.vt_codes = vt_codes;
    a.q_sf = ws + L.q_sf;
    a.k_sf = ws + L.k_sf;
    a.v_sf = ws + L.v_sf;
    a.O = O;
    a.status = status;
    a.BH = BH;
    a.N = N;
    a.d = d;
    a.kv_tile = kv_tile;
    a.pnq = pnq;
    a.qmax = q;
    a.softmax_scale = resolve_scale(softmax_scale, d);
    e = mxattn::launch_attention(a, s);
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_workspace_status(const void* workspace, mxattn_stream_t stream) {
    if (workspace == nullptr) return MXATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return MXATTN_ERR_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MXATTN_ERR_CUDA;
    return (word & 4u) ? MXATTN_ERR_TIMEOUT : MXATTN_OK;
}

// ------------------------------------------------------------------ NVFP4 comparison variant

namespace {

struct NvLayout {
    size_t status, q_codes, k_codes, vt_codes, q_sf, k_sf, v_sf, amax, gs, total;
};

bool make_layout_nv(int B, int H, int N, int d, NvLayout* L) {
    if (B < 1 || H < 1 || N < 1 || N > kMaxN || (d != 64 && d != 128)) return false;
    const size_t BH = static_cast<size_t>(B) * H;
    const size_t G = (static_cast<size_t>(N) + 127) / 128;
    const size_t npad = (static_cast<size_t>(N) + 31) / 32 * 32;
    size_t off = 0;
    L->status = off;
    off += 256;
    L->q_codes = off;
    off = align256(off + BH * N * d / 2);
    L->k_codes = off;
    off = align256(off + BH * N * d / 2);
    L->vt_codes = off;
    off = align256(off + BH * d * npad / 2);
    L->q_sf = off;
    off = align256(off + BH * G * (d / 64) * 512);
    L->k_sf = off;
    off = align256(off + BH * G * (d / 64) * 512);
    L->v_sf = off;
    off = align256(off + BH * G * 1024);
    L->amax = off;
    off = align256(off + 3 * BH * 4);
    L->gs = off;
    off = align256(off + 3 * BH * 4);
    L->total = off;
    return true;
}

mxattn_status check_nv_args(int B, int H, int N, int d, int kv_tile, int pnq, const float* O, const void* ws,
                            size_t ws_bytes, NvLayout* L) {
    if (B < 1 || H < 1 || N < 1 || O == nullptr || ws == nullptr) return MXATTN_ERR_INVALID;
    if (pnq != 0 && pnq != 1) return MXATTN_ERR_INVALID;
    if (d != 64 && d != 128) return MXATTN_ERR_UNSUPPORTED;
    if (kv_tile != 64 && kv_tile != 128) return MXATTN_ERR_UNSUPPORTED;
    if (N > kMaxN || static_cast<int64_t>(B) * H > 65535) return MXATTN_ERR_UNSUPPORTED;
    if (!make_layout_nv(B, H, N, d, L)) return MXATTN_ERR_INVALID;
    if (ws_bytes < L->total || !aligned(ws, 256) || !aligned(O, 16)) return MXATTN_ERR_INVALID;
    return MXATTN_OK;
}

}  // namespace

MXATTN_API size_t mxattn_nvfp4_workspace_size(int B, int H, int N, int d) {
    NvLayout L;
    return make_layout_nv(B, H, N, d, &L) ? L.total : 0;
}

MXATTN_API mxattn_status mxattn_nvfp4_quantize(const void* x, int64_t rows, int64_t cols, uint8_t* codes,
                                               uint8_t* scales, float* gs, mxattn_stream_t stream) {
    if (rows < 0 || cols <= 0 || cols % 16 != 0) return MXATTN_ERR_INVALID;
    if (rows == 0) return MXATTN_OK;  // nothing to do
    if (x == nullptr || codes == nullptr || scales == nullptr || gs == nullptr) return MXATTN_ERR_INVALID;
    if (!aligned(x, 16) || !aligned(codes, 4) || !aligned(gs, 4)) return MXATTN_ERR_INVALID;
    cudaError_t e = mxattn::launch_nv_quantize_rows(x, rows, cols, codes, scales, gs,
                                                     reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_nvfp4_prepare(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                              void* workspace, size_t workspace_bytes, mxattn_stream_t stream) {
    NvLayout L;
    float dummy_out[4];
    mxattn_status st = check_nv_args(B, H, N, d, 128, 1, dummy_out, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    if (Q == nullptr || K == nullptr || V == nullptr) return MXATTN_ERR_INVALID;
    if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16)) return MXATTN_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t BH = static_cast<int64_t>(B) * H;
    const int G = (N + 127) / 128;
    uint32_t* amax = reinterpret_cast<uint32_t*>(ws + L.amax);
    float* gs = reinterpret_cast<float*>(ws + L.gs);
    cudaError_t e = mxattn::launch_nv_amax(Q, K, V, 3, static_cast<int64_t>(N) * d, BH, amax, s);
    if (e != cudaSuccess) return MXATTN_ERR_CUDA;
    e = mxattn::launch_nv_quantize_qk(Q, K, ws + L.q_codes, ws + L.k_codes, ws + L.q_sf, ws + L.k_sf, amax, amax + BH,
                                      gs, gs + BH, BH, N, d, G, reinterpret_cast<uint32_t*>(ws + L.status), s);
    if (e != cudaSuccess) return MXATTN_ERR_CUDA;
    e = mxattn::launch_nv_quantize_vt(V, BH, N, d, G, amax + 2 * BH, gs + 2 * BH, ws + L.vt_codes, ws + L.v_sf, s);
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_nvfp4_attend(int B, int H, int N, int d, int kv_tile, int pnq, float softmax_scale,
                                             float* O, void* workspace, size_t workspace_bytes,
                                             mxattn_stream_t stream) {
    NvLayout L;
    mxattn_status st = check_nv_args(B, H, N, d, kv_tile, pnq, O, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    mxattn::AttnArgs a{};
    a.q_codes = ws + L.q_codes;
    a.k_codes = ws + L.k_codes;
    a.vt_codes = ws + L.vt_codes;
    a.q_sf = ws + L.q_sf;
    a.k_sf = ws + L.k_sf;
    a.v_sf = ws + L.v_sf;
    a.O = O;
    a.status = reinterpret_cast<uint32_t*>(ws + L.status);
    a.BH = static_cast<int64_t>(B) * H;
    a.N = N;
    a.d = d;
    a.kv_tile = kv_tile;
    a.pnq = pnq;
    a.qmax = 8.f;  // unused by the NVFP4 path
    a.softmax_scale = resolve_scale(softmax_scale, d);
    a.nv = 1;
    a.gs = reinterpret_cast<const float*>(ws + L.gs);
    cudaError_t e = mxattn::launch_attention(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

MXATTN_API mxattn_status mxattn_nvfp4_forward(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                              int kv_tile, int pnq, float softmax_scale, float* O, void* workspace,
                                              size_t workspace_bytes, mxattn_stream_t stream) {
    NvLayout L;
    mxattn_status st = check_nv_args(B, H, N, d, kv_tile, pnq, O, workspace, workspace_bytes, &L);
    if (st != MXATTN_OK) return st;
    st = mxattn_nvfp4_prepare(Q, K, V, B, H, N, d, workspace, workspace_bytes, stream);
    if (st != MXATTN_OK) return st;
    return mxattn_nvfp4_attend(B, H, N, d, kv_tile, pnq, softmax_scale, O, workspace, workspace_bytes, stream);
}
