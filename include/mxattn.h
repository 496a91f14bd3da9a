/*
 * mxattn.h -- C ABI of libmxattn.so: MXFP4 attention with Universal Optimal
 * Scaling (UOS) and Pre-Normalization Quantization (PNQ) on NVIDIA B200
 * (sm_100a).
 *
 * Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 * Quantization for MXFP4 Attention", abstract.  It fixes the MXFP4 operand
 * format ("OCP MXFP4", power-of-two microscaling), the UOS scaling boundary
 * Qmax = 7.25, and PNQ: the unnormalized softmax exponentials are quantized
 * before the row-wise sum, so the sum is built from the same quantized values
 * that weight V.  Readings of what the abstract leaves open:
 *   - MXFP4 blocks are 32 consecutive elements along the contraction axis of
 *     each product (Q, K: along the head dimension d; P: along keys, aligned
 *     to key-tile starts; V: along tokens), with E2M1 elements
 *     {0, .5, 1, 1.5, 2, 3, 4, 6} x sign and one E8M0 scale 2^e per block.
 *   - OCP rule: e = floor(log2 amax) - 2.  UOS rule: the smallest e with
 *     amax <= 7.25 * 2^e.  Both clamp e to [-127, 127]; amax = 0 gives -127.
 *   - Elements round to nearest, ties to the even code, saturating at 6; the
 *     sign of a value that rounds to zero is kept (code 0x8).
 *   - The softmax scale is applied to the fp32 product of the dequantized Q
 *     and K; the online softmax walks key tiles of kv_tile columns in
 *     ascending order and subtracts the running maximum after each tile.
 *   - PNQ off: P*V still uses the quantized exponentials but the row sum uses
 *     the unquantized ones (the error in the row-wise normalization that the abstract names).
 *
 * Conventions for every entry point:
 *   - Pointers are device pointers unless stated otherwise; the caller owns
 *     every buffer, including the workspace.  The library allocates no device
 *     memory and keeps no state between calls except cached function handles.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are returned synchronously and launch
 *     nothing.  MXATTN_ERR_CUDA reports a launch error (cudaGetLastError).
 *   - Layouts are row-major and contiguous.  A code byte holds element 2i in
 *     its low nibble and element 2i+1 in its high nibble.  A scale byte is
 *     the E8M0 encoding e + 127.
 *   - bf16 inputs are IEEE bfloat16 bit patterns; NaN and Inf inputs are
 *     outside the contract (the result is unspecified but the call is safe).
 */
#ifndef MXATTN_H
#define MXATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* mxattn_stream_t;

typedef enum {
    MXATTN_OK = 0,
    MXATTN_ERR_INVALID = 1,     /* null pointer, negative or inconsistent size, small workspace */
    MXATTN_ERR_UNSUPPORTED = 2, /* d or kv_tile outside the supported set, N too large */
    MXATTN_ERR_CUDA = 3,        /* a CUDA launch or driver call failed */
    MXATTN_ERR_TIMEOUT = 4      /* a bounded wait inside the attention kernel gave up (read via
                                   mxattn_workspace_status) */
} mxattn_status;

typedef enum {
    MXATTN_RULE_OCP = 0, /* e = floor(log2 amax) - 2 */
    MXATTN_RULE_UOS = 1  /* smallest e with amax <= 7.25 * 2^e (the abstract's Qmax) */
} mxattn_rule;

/*
 * Scale boundary Qmax.  The abstract names the UOS scaling boundary Qmax and
 * chooses 7.25; the *_qmax entry points below take any boundary in (4, 8] for
 * the same rule -- e = the smallest integer with amax <= qmax * 2^e, clamped
 * to [-127, 127] -- so the boundary can be swept.  qmax = 8 selects the OCP
 * rule e = floor(log2 amax) - 2, which the boundary rule approaches as qmax
 * tends to 8 from below.  MXATTN_RULE_UOS is qmax = 7.25 and MXATTN_RULE_OCP
 * is qmax = 8: every rule-taking call equals its *_qmax form at that value.
 * A qmax outside (4, 8] (or NaN) returns MXATTN_ERR_INVALID.
 */

/*
 * Standalone MXFP4 quantize/pack (the abstract's direct MXFP4 quantization;
 * the scale rule is UOS or OCP).
 *   x:      bf16 [rows, cols], cols % 32 == 0, 16-byte aligned.
 *   codes:  u8 [rows, cols/2] (packed E2M1), 4-byte aligned.
 *   scales: u8 [rows, cols/32] (E8M0), one per 32-element block.
 * rows == 0 is a no-op.  Errors: MXATTN_ERR_INVALID for null pointers,
 * negative sizes, cols % 32 != 0 or misaligned pointers.
 */
mxattn_status mxattn_quantize(const void* x, int64_t rows, int64_t cols, mxattn_rule rule,
                              uint8_t* codes, uint8_t* scales, mxattn_stream_t stream);

/* mxattn_quantize with a scale boundary qmax in (4, 8] instead of a named rule. */
mxattn_status mxattn_quantize_qmax(const void* x, int64_t rows, int64_t cols, float qmax, uint8_t* codes,
                                   uint8_t* scales, mxattn_stream_t stream);

/*
 * V quantize with transpose: blocks of 32 consecutive tokens of each channel
 * (reading: the scale runs along the contraction axis of P*V).
 *   v:        bf16 [BH, N, d], d in {64, 128}, 16-byte aligned.
 *   codes_t:  u8 [BH, d, Npad/2], Npad = ceil(N/32)*32; tokens >= N are zeros.
 *   scales_t: u8 [BH, d, Npad/32].
 * Errors: MXATTN_ERR_INVALID (null, N < 1, BH < 1), MXATTN_ERR_UNSUPPORTED (d).
 */
mxattn_status mxattn_quantize_vt(const void* v, int64_t BH, int64_t N, int64_t d, mxattn_rule rule,
                                 uint8_t* codes_t, uint8_t* scales_t, mxattn_stream_t stream);

/*
 * Bytes of workspace that mxattn_forward / mxattn_forward_quantized need for
 * this shape (0 for invalid shapes).  With G = ceil(N/128), Npad =
 * ceil(N/32)*32 and every region starting on a 256-byte boundary, the
 * workspace holds, in order:
 *   status   256 bytes (u32 error word of the last forward on this workspace)
 *   q_codes  B*H*N*d/2      k_codes  B*H*N*d/2      vt_codes B*H*d*Npad/2
 *   q_sf     B*H*G*512      k_sf     B*H*G*512      vt_sf    B*H*G*512
 * The *_codes regions use the layouts of mxattn_quantize / mxattn_quantize_vt.
 * The *_sf regions hold the E8M0 scales regrouped per 128 rows (Q, K) or 128
 * tokens (V^T): within a group, row m (or channel m of V^T) and block k sit at
 * byte (m%32)*16 + (m/32)*4 + k -- the order in which the tensor core reads
 * scale factors -- with rows past N set to 0 and unused V^T channel rows to
 * 127.
 */
size_t mxattn_workspace_size(int B, int H, int N, int d);

/*
 * Fused MXFP4 attention forward, non-causal:
 *   O = softmax(deq(Qq) deq(Kq)^T * softmax_scale) with MXFP4 P, times deq(Vq),
 * evaluated as the tile-ordered online softmax described above.
 *   Q, K, V: bf16 [B, H, N, d], 16-byte aligned.  O: fp32 [B, H, N, d], 16-byte aligned.
 *   d in {64, 128}; kv_tile in {64, 128}; 1 <= N <= 2^24; pnq in {0, 1};
 *   rule applies to Q, K, V and P; softmax_scale <= 0 selects 1/sqrt(d).
 *   workspace: >= mxattn_workspace_size(B, H, N, d) bytes, 256-byte aligned.
 * Launches two kernels on `stream`: the operand preparation (Q, K and V^T
 * quantized in one launch) and the attention.  Both kernels' waits are
 * bounded; if one gives up it records MXATTN_ERR_TIMEOUT in the workspace
 * status word (see mxattn_workspace_status) and O is unspecified.
 */
mxattn_status mxattn_forward(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                             int kv_tile, int pnq, mxattn_rule rule, float softmax_scale, float* O,
                             void* workspace, size_t workspace_bytes, mxattn_stream_t stream);

/*
 * mxattn_forward in two calls, for callers that time or schedule the steps
 * separately: mxattn_prepare launches the operand preparation (Q, K and V^T
 * quantized in one kernel) into the workspace and resets its status word;
 * mxattn_attend launches the
 * attention kernel on a workspace that mxattn_prepare filled for the same
 * (B, H, N, d) and `rule`.  mxattn_forward == mxattn_prepare + mxattn_attend.
 * Same constraints and errors as mxattn_forward.
 */
mxattn_status mxattn_prepare(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                             mxattn_rule rule, void* workspace, size_t workspace_bytes, mxattn_stream_t stream);
mxattn_status mxattn_attend(int B, int H, int N, int d, int kv_tile, int pnq, mxattn_rule rule, float softmax_scale,
                            float* O, void* workspace, size_t workspace_bytes, mxattn_stream_t stream);

/*
 * mxattn_forward / mxattn_prepare / mxattn_attend with a scale boundary qmax in
 * (4, 8] for Q, K, V and P instead of a named rule.  Same arguments, layouts,
 * constraints and errors otherwise; mxattn_attend_qmax must run on a workspace
 * that mxattn_prepare_qmax filled with the same qmax.
 */
mxattn_status mxattn_forward_qmax(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                  int kv_tile, int pnq, float qmax, float softmax_scale, float* O, void* workspace,
                                  size_t workspace_bytes, mxattn_stream_t stream);
mxattn_status mxattn_prepare_qmax(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                  float qmax, void* workspace, size_t workspace_bytes, mxattn_stream_t stream);
mxattn_status mxattn_attend_qmax(int B, int H, int N, int d, int kv_tile, int pnq, float qmax, float softmax_scale,
                                 float* O, void* workspace, size_t workspace_bytes, mxattn_stream_t stream);

/*
 * The attention step alone, on operands already quantized by the caller in
 * the public layouts: q_codes/k_codes u8 [B,H,N,d/2], q_scales/k_scales u8
 * [B,H,N,d/32] (as mxattn_quantize), vt_codes u8 [B,H,d,Npad/2], vt_scales u8
 * [B,H,d,Npad/32] (as mxattn_quantize_vt).  `rule` is the rule for P.  The
 * scales are regrouped into the workspace's *_sf regions first (the codes
 * regions of the workspace are not used).  Same constraints and errors as
 * mxattn_forward; code pointers 16-byte aligned.
 */
mxattn_status mxattn_forward_quantized(const uint8_t* q_codes, const uint8_t* q_scales, const uint8_t* k_codes,
                                       const uint8_t* k_scales, const uint8_t* vt_codes, const uint8_t* vt_scales,
                                       int B, int H, int N, int d, int kv_tile, int pnq, mxattn_rule rule,
                                       float softmax_scale, float* O, void* workspace, size_t workspace_bytes,
                                       mxattn_stream_t stream);

/*
 * mxattn_forward from host buffers to host buffers, with the transfers
 * overlapped against the attention (a deployment entry point; the paper has
 * no counterpart).  The (batch, head) slices are independent, so they are
 * processed in groups: the copy to the device of group i+1 (one
 * cudaMemcpyAsync each for Q, K, V) and the copy back of group i-1 overlap
 * the attention of group i (one mxattn_forward per group on `stream`).
 *   Q, K, V:   HOST bf16 [B, H, N, d]; O: HOST fp32 [B, H, N, d].  Page-locked
 *              (pinned) host memory lets the copies run asynchronously; with
 *              pageable memory the call still works but the copies do not
 *              overlap.
 *   q_dev, k_dev, v_dev: device bf16 [B, H, N, d] staging buffers, o_dev:
 *              device fp32 [B, H, N, d], each 16-byte aligned.
 *   workspace: device, 256-byte aligned, at least
 *              mxattn_forward_host_workspace_size(B, H, N, d, group_sizes,
 *              ngroups) bytes (the workspace of the largest group); its
 *              status word holds the last group's timeout status
 *              (mxattn_workspace_status).
 *   group_sizes: NULL, or ngroups positive group sizes (in slices) that sum
 *              to B*H, processed in order.  With NULL, ngroups groups
 *              (0: 16; at most B*H): the first and the last of one slice each
 *              (the only transfers nothing overlaps), the rest as equal as
 *              possible.
 * The copies run on two streams the call creates (one per direction); events
 * order them against `stream`, which waits for the last copy back: when
 * `stream` reaches the point after this call, O holds the result.  The
 * streams and events are released by the runtime once that work is done.
 * Argument errors as mxattn_forward, plus MXATTN_ERR_INVALID for a null or
 * misaligned buffer, bad group sizes or a small workspace; MXATTN_ERR_CUDA if
 * a stream, event or copy call fails (work already enqueued stays ordered
 * before later work on `stream`).
 */
size_t mxattn_forward_host_workspace_size(int B, int H, int N, int d, const int* group_sizes, int ngroups);
mxattn_status mxattn_forward_host(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                  int kv_tile, int pnq, mxattn_rule rule, float softmax_scale, float* O,
                                  void* q_dev, void* k_dev, void* v_dev, float* o_dev, void* workspace,
                                  size_t workspace_bytes, const int* group_sizes, int ngroups,
                                  mxattn_stream_t stream);

/*
 * mxattn_forward without a caller-provided workspace, for callers that cannot
 * allocate device memory themselves: code embedded in a host framework that
 * owns all device memory through its own pool and forbids raw cudaMalloc, or
 * a latency-critical loop that must not pay for cudaMalloc's implicit device
 * synchronization.  (The MXAttention paper has no counterpart; this is a
 * deployment convenience.)
 *   - The workspace is a fixed 16 MiB array of device memory inside this
 *     library's CUDA module; every device that loads the library holds it
 *     until the process exits.  Shapes whose mxattn_workspace_size exceeds
 *     16 MiB (16777216 bytes) are rejected with MXATTN_ERR_UNSUPPORTED before
 *     anything is launched.  The call itself allocates and frees nothing.
 *   - The first call on a device looks up the array's device address (once
 *     per device); make that first call before any stream capture.
 *   - All calls share the one array, and it keeps the last call's contents
 *     (each call rewrites what it reads, including the status word).  Calls
 *     that may overlap on the GPU -- on different streams, or from different
 *     threads -- race on it; serialize them.
 *   - The kernels' timeout status is not reported by this call (a bounded
 *     wait that gives up leaves O unspecified); use mxattn_forward with a
 *     workspace and mxattn_workspace_status when that status is needed.
 * Arguments, constraints and other errors as mxattn_forward.
 */
mxattn_status mxattn_forward_noalloc(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                     int kv_tile, int pnq, mxattn_rule rule, float softmax_scale, float* O,
                                     mxattn_stream_t stream);

/*
 * Synchronizes `stream`, reads the status word of `workspace` (written by
 * the last forward that used it) and returns MXATTN_OK or
 * MXATTN_ERR_TIMEOUT.  MXATTN_ERR_CUDA if the synchronization or copy fails.
 * The word is reset by the next forward on this workspace.
 */
mxattn_status mxattn_workspace_status(const void* workspace, mxattn_stream_t stream);

/*
 * Failure-detection self-test of the bounded wait that every mbarrier wait in
 * the attention kernel goes through (this library's own safeguard; the paper
 * has no counterpart).  Launches one warp on `stream` that waits on a shared
 * memory mbarrier for phase 0 with a limit of `timeout_us` microseconds
 * (1 .. 1,000,000).  If `arrive` is non-zero the barrier's single arrival is
 * made first and the wait completes at once; otherwise nobody arrives and the
 * wait gives up at its limit, raising the kernel's abort flag.  Nothing
 * faults: the kernel returns either way and the context stays usable.
 *   out: device u32[3], 4-byte aligned, written by the kernel:
 *        out[0] = 0 (completed) or MXATTN_ERR_TIMEOUT (gave up),
 *        out[1] = microseconds the warp spent waiting,
 *        out[2] = bit 0 abort flag raised, bit 1 wait left without completion.
 * Returns MXATTN_ERR_INVALID (null/misaligned out, timeout out of range) or
 * MXATTN_ERR_CUDA (launch failed); otherwise MXATTN_OK (asynchronous: read
 * `out` after synchronizing `stream`).
 */
mxattn_status mxattn_wait_selftest(int arrive, unsigned timeout_us, unsigned* out, mxattn_stream_t stream);

/* ---------------------------------------------------------------------------
 * NVFP4 comparison variant.  The abstract measures MXAttention against
 * NVFP4 baselines without defining them; this library's reading is
 * NVIDIA's NVFP4 applied to the same four operands and the same softmax loop:
 *   - E2M1 elements (as above) in blocks of 16 along the contraction axis,
 *     one unsigned E4M3 (OCP FP8 E4M3) scale per block, and one fp32
 *     second-level scale per (batch, head) slice of Q, K or V;
 *   - g = 448 / max(amax_slice, 2^-100), block scale sb = E4M3(amax_block * g)
 *     (round to nearest even, saturating at 448), element code
 *     E2M1(x * ((6 g) / sb)), all in fp32 with round to nearest; a block whose
 *     scale rounds to 0 holds zeros (sign kept); value = code * sb / (6 g);
 *   - P (<= 1 by construction) uses g = 448 with blocks of 16 keys aligned to
 *     key-tile starts; PNQ on/off as for MXFP4.
 * Codes and scales decided from bf16 inputs are exact functions of these
 * definitions (no approximation): the oracle reproduces them bit for bit.
 * The tensor-core step is tcgen05.mma kind::mxf4nvf4 (block16, E4M3 scales).
 * ------------------------------------------------------------------------- */

/*
 * Standalone NVFP4 quantization of a whole tensor (one second-level scale):
 *   x:      bf16 [rows, cols], cols % 16 == 0, 16-byte aligned.
 *   codes:  u8 [rows, cols/2] (4-byte aligned).  scales: u8 [rows, cols/16] E4M3.
 *   gs:     device float[2], 4-byte aligned, written by the call: gs[0] = amax
 *           of x, gs[1] = g = 448 / max(amax, 2^-100).
 * Launches an amax pass, the quantizer and a one-thread kernel that stores g;
 * rows == 0 launches nothing and returns MXATTN_OK.
 * Errors: MXATTN_ERR_INVALID (null, misaligned, rows < 0, cols not a positive
 * multiple of 16), MXATTN_ERR_CUDA (launch failed).
 */
mxattn_status mxattn_nvfp4_quantize(const void* x, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                                    float* gs, mxattn_stream_t stream);

/*
 * Workspace bytes for the NVFP4 forward (0 for invalid shapes).  Regions, each
 * on a 256-byte boundary, in order (G = ceil(N/128), Npad = ceil(N/32)*32):
 *   status 256 bytes (u32 error word, as for the MXFP4 workspace)
 *   q_codes B*H*N*d/2   k_codes B*H*N*d/2   vt_codes B*H*d*Npad/2
 *   q_sf    B*H*G*(d/64)*512   k_sf B*H*G*(d/64)*512   vt_sf B*H*G*1024
 *   amax    3*B*H u32 (fp32 bits of |Q|, |K|, |V| maxima per (b, h))
 *   g       3*B*H fp32 (second-level scales of Q, K, V per (b, h))
 * Scale regions are regrouped per 128 rows (Q, K) or 128 tokens (V^T) and
 * per 64 columns of the contraction axis: 512-byte atoms in which row m (or
 * channel m) and 16-element block b of the 64 columns sit at byte
 * (m%32)*16 + (m/32)*4 + b; rows past N hold 0, unused V^T channel rows 0x38
 * (E4M3 1.0).
 */
size_t mxattn_nvfp4_workspace_size(int B, int H, int N, int d);

/*
 * NVFP4 attention forward (non-causal), the same tile-ordered online softmax
 * as mxattn_forward with every operand in NVFP4:
 *   Q, K, V: bf16 [B, H, N, d], 16-byte aligned.  O: fp32 [B, H, N, d].
 *   d in {64, 128}; kv_tile in {64, 128}; 1 <= N <= 2^24; B*H <= 65535;
 *   pnq in {0, 1}; softmax_scale <= 0 selects 1/sqrt(d).
 *   workspace: >= mxattn_nvfp4_workspace_size(B, H, N, d) bytes, 256-byte aligned.
 * mxattn_nvfp4_prepare launches the amax pass and the Q/K and V^T quantizers
 * into the workspace; mxattn_nvfp4_attend runs the attention kernel on it;
 * mxattn_nvfp4_forward is the two in order.  The status word and
 * mxattn_workspace_status work as for the MXFP4 workspace.
 * Errors as mxattn_forward.
 */
mxattn_status mxattn_nvfp4_forward(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                   int kv_tile, int pnq, float softmax_scale, float* O, void* workspace,
                                   size_t workspace_bytes, mxattn_stream_t stream);
mxattn_status mxattn_nvfp4_prepare(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                   void* workspace, size_t workspace_bytes, mxattn_stream_t stream);
mxattn_status mxattn_nvfp4_attend(int B, int H, int N, int d, int kv_tile, int pnq, float softmax_scale, float* O,
                                  void* workspace, size_t workspace_bytes, mxattn_stream_t stream);

/*
 * Self-test of the softmax's decisions on P (this library's own check; the
 * paper has no counterpart).  Runs, on n inputs, the device functions the
 * attention kernel uses for P, so they can be compared with a reference:
 *   path 0, 1, 2: in = w (fp32), out = E2M1 code (0..15) of 2^w computed by
 *     ex2.approx (0), by the FMA-pipe code-only stand-in used with PNQ (1;
 *     its input map u = sat((w + 2) / 8) included), or by the FMA-pipe
 *     degree-5 exponential used without PNQ (2), each rounded by
 *     cvt.rn.satfinite.e2m1x2;
 *   path 3: in = x (log2 of a block's largest exponential, <= 0), out = the
 *     MXFP4 block exponent e for the scale boundary qmax in (4, 8] (8 = OCP);
 *   path 4: in = x, out = the NVFP4 block scale byte E4M3(2^x * 448);
 *   path 5: in = v, out = E2M1 code (0..15) of v by cvt.rn.satfinite.e2m1x2
 *     alone (the rounding step every path ends with).
 *   in: device fp32 [n], out: device i32 [n], both 4-byte aligned; n % 8 == 0.
 * Errors: MXATTN_ERR_INVALID (path, n, qmax for path 3, null or misaligned
 * pointers), MXATTN_ERR_CUDA (launch failed).  Asynchronous on `stream`.
 */
mxattn_status mxattn_p_selftest(int path, const float* in, int64_t n, float qmax, int32_t* out,
                                mxattn_stream_t stream);

/*
 * Measurement utility (this library's own; the paper has no counterpart): the
 * throughput ceiling of the block-scaled FP4 tensor-core instruction the
 * attention kernel uses.  Launches `ctas` CTAs; in each, one thread issues
 * 2 * iters tcgen05.mma.kind::mxf4.block_scale.block32 instructions of shape
 * M = 128, N = 128, K = 64 (the attention kernel's S = Q K^T shape and
 * descriptors) back to back on operands held in shared memory, accumulating
 * into one TMEM tile.  Work per launch: ctas * iters * 2 * (2 * 128 * 128 * 64)
 * flop; time it with events on `stream`.
 *   ctas in [1, 4096], iters in [1, 200000] (a launch then takes milliseconds);
 *   status: device u32, 4-byte aligned; zeroed by the call, MXATTN_ERR_TIMEOUT
 *     ORed in if the final wait gave up (2 s).
 *   cycles: device u64 [ctas], 8-byte aligned, or NULL; CTA i writes the SM
 *     clock cycles from its first issue to the completion of its last MMA, so
 *     the rate per clock (2 * iters * 2 * 128 * 128 * 64 / cycles per SM, with
 *     one CTA per SM) does not depend on the clock the power cap allows.
 * Errors: MXATTN_ERR_INVALID (arguments), MXATTN_ERR_CUDA (launch failed).
 * Asynchronous on `stream`.
 */
mxattn_status mxattn_mxf4_mma_loop(int ctas, int iters, uint32_t* status, uint64_t* cycles,
                                   mxattn_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char* mxattn_status_string(mxattn_status status);

#ifdef __cplusplus
}
#endif

#endif /* MXATTN_H */
