"""ctypes binding of libmxattn.so (C ABI in include/mxattn.h).

The functions carry the C names and only marshal arguments: torch tensors in,
raw device pointers and sizes out, the current CUDA stream passed through.
All compute happens in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxattn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "mxattn.h")

STATUS = {0: "MXATTN_OK", 1: "MXATTN_ERR_INVALID", 2: "MXATTN_ERR_UNSUPPORTED", 3: "MXATTN_ERR_CUDA",
          4: "MXATTN_ERR_TIMEOUT"}
RULES = {"ocp": 0, "uos": 1}


class MxattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmxattn.so (raises if it was not built: there is no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mxfp4_microscaled_quantization_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, i32, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.mxattn_status_string.argtypes = [i32]
        L.mxattn_status_string.restype = ctypes.c_char_p
        L.mxattn_quantize.argtypes = [P, i64, i64, i32, P, P, P]
        L.mxattn_quantize.restype = i32
        L.mxattn_quantize_vt.argtypes = [P, i64, i64, i64, i32, P, P, P]
        L.mxattn_quantize_vt.restype = i32
        L.mxattn_workspace_size.argtypes = [i32, i32, i32, i32]
        L.mxattn_workspace_size.restype = u64
        L.mxattn_forward.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float, P, P, u64, P]
        L.mxattn_forward.restype = i32
        L.mxattn_prepare.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, u64, P]
        L.mxattn_prepare.restype = i32
        L.mxattn_attend.argtypes = [i32, i32, i32, i32, i32, i32, i32, ctypes.c_float, P, P, u64, P]
        L.mxattn_attend.restype = i32
        L.mxattn_forward_quantized.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32,
                                               ctypes.c_float, P, P, u64, P]
        L.mxattn_forward_quantized.restype = i32
        L.mxattn_forward_noalloc.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float, P, P]
        L.mxattn_forward_noalloc.restype = i32
        L.mxattn_forward_host_workspace_size.argtypes = [i32, i32, i32, i32, P, i32]
        L.mxattn_forward_host_workspace_size.restype = u64
        L.mxattn_forward_host.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float, P, P, P, P, P, P,
                                          u64, P, i32, P]
        L.mxattn_forward_host.restype = i32
        f32 = ctypes.c_float
        L.mxattn_quantize_qmax.argtypes = [P, i64, i64, f32, P, P, P]
        L.mxattn_quantize_qmax.restype = i32
        L.mxattn_forward_qmax.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f32, f32, P, P, u64, P]
        L.mxattn_forward_qmax.restype = i32
        L.mxattn_prepare_qmax.argtypes = [P, P, P, i32, i32, i32, i32, f32, P, u64, P]
        L.mxattn_prepare_qmax.restype = i32
        L.mxattn_attend_qmax.argtypes = [i32, i32, i32, i32, i32, i32, f32, f32, P, P, u64, P]
        L.mxattn_attend_qmax.restype = i32
        L.mxattn_workspace_status.argtypes = [P, P]
        L.mxattn_workspace_status.restype = i32
        L.mxattn_wait_selftest.argtypes = [i32, ctypes.c_uint, P, P]
        L.mxattn_wait_selftest.restype = i32
        L.mxattn_p_selftest.argtypes = [i32, P, i64, f32, P, P]
        L.mxattn_p_selftest.restype = i32
        L.mxattn_mxf4_mma_loop.argtypes = [i32, i32, P, P, P]
        L.mxattn_mxf4_mma_loop.restype = i32
        L.mxattn_nvfp4_quantize.argtypes = [P, i64, i64, P, P, P, P]
        L.mxattn_nvfp4_quantize.restype = i32
        L.mxattn_nvfp4_workspace_size.argtypes = [i32, i32, i32, i32]
        L.mxattn_nvfp4_workspace_size.restype = u64
        L.mxattn_nvfp4_forward.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f32, P, P, u64, P]
        L.mxattn_nvfp4_forward.restype = i32
        L.mxattn_nvfp4_prepare.argtypes = [P, P, P, i32, i32, i32, i32, P, u64, P]
        L.mxattn_nvfp4_prepare.restype = i32
        L.mxattn_nvfp4_attend.argtypes = [i32, i32, i32, i32, i32, i32, f32, P, P, u64, P]
        L.mxattn_nvfp4_attend.restype = i32
        _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Names of the entry points declared in include/mxattn.h."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(mxattn_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().mxattn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise MxattnError(status, where)


def _rule(rule) -> int:
    if not isinstance(rule, str):
        raise ValueError(f"this call takes a named rule ('ocp' or 'uos'), got {rule!r}")
    return RULES[rule]


def _qmax(rule):
    """None for a named rule ('ocp', 'uos'); else the scale boundary Qmax in (4, 8]
    (checked by the library) for the *_qmax entry points."""
    return None if isinstance(rule, str) else float(rule)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def mxattn_quantize(x: torch.Tensor, rule="uos", codes=None, scales=None, stream=None):
    """bf16 [..., cols] -> (codes u8 [..., cols/2], scales u8 [..., cols/32])."""
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (cols // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (cols // 32,), dtype=torch.uint8, device=x.device)
    q = _qmax(rule)
    if q is None:
        _check(lib().mxattn_quantize(_cuda(x, "x", torch.bfloat16), rows, cols, _rule(rule), _cuda(codes, "codes"),
                                     _cuda(scales, "scales"), _stream(stream)), "mxattn_quantize")
    else:
        _check(lib().mxattn_quantize_qmax(_cuda(x, "x", torch.bfloat16), rows, cols, q, _cuda(codes, "codes"),
                                          _cuda(scales, "scales"), _stream(stream)), "mxattn_quantize_qmax")
    return codes, scales


def mxattn_quantize_vt(v: torch.Tensor, rule="uos", codes_t=None, scales_t=None, stream=None):
    """V bf16 [..., N, d] -> V^T (codes u8 [..., d, Npad/2], scales u8 [..., d, Npad/32])."""
    N, d = v.shape[-2:]
    BH = v.numel() // (N * d)
    npad = (N + 31) // 32 * 32
    lead = tuple(v.shape[:-2])
    if codes_t is None:
        codes_t = torch.empty(lead + (d, npad // 2), dtype=torch.uint8, device=v.device)
    if scales_t is None:
        scales_t = torch.empty(lead + (d, npad // 32), dtype=torch.uint8, device=v.device)
    _check(lib().mxattn_quantize_vt(_cuda(v, "v", torch.bfloat16), BH, N, d, _rule(rule), _cuda(codes_t, "codes_t"),
                                    _cuda(scales_t, "scales_t"), _stream(stream)), "mxattn_quantize_vt")
    return codes_t, scales_t


def mxattn_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib().mxattn_workspace_size(B, H, N, d))


def workspace_layout(B: int, H: int, N: int, d: int) -> dict:
    """Byte offsets of the workspace regions (as documented in include/mxattn.h)."""
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    BH, G, npad = B * H, (N + 127) // 128, (N + 31) // 32 * 32
    off, out = 0, {}
    for name, size in (("status", 256), ("q_codes", BH * N * d // 2), ("k_codes", BH * N * d // 2),
                       ("vt_codes", BH * d * npad // 2), ("q_sf", BH * G * 512), ("k_sf", BH * G * 512),
                       ("vt_sf", BH * G * 512)):
        out[name] = (off, size)
        off = a(off + size)
    out["total"] = off
    return out


def new_workspace(B, H, N, d, device="cuda") -> torch.Tensor:
    n = mxattn_workspace_size(B, H, N, d)
    if n == 0:
        raise MxattnError(1, "mxattn_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def mxattn_forward(q, k, v, kv_tile=128, pnq=True, rule="uos", softmax_scale=0.0, out=None, workspace=None,
                   stream=None):
    """Fused MXFP4 attention: q, k, v bf16 [B, H, N, d] -> O fp32 [B, H, N, d].
    `rule`: "uos", "ocp", or a scale boundary Qmax in (4, 8] (mxattn_forward_qmax)."""
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, H, N, d, q.device)
    qm = _qmax(rule)
    fn, name = (lib().mxattn_forward, "mxattn_forward") if qm is None else (lib().mxattn_forward_qmax,
                                                                             "mxattn_forward_qmax")
    _check(fn(_cuda(q, "q", torch.bfloat16), _cuda(k, "k", torch.bfloat16), _cuda(v, "v", torch.bfloat16), B, H, N, d,
              kv_tile, 1 if pnq else 0, _rule(rule) if qm is None else qm, float(softmax_scale),
              _cuda(out, "out", torch.float32), _cuda(workspace, "workspace"), workspace.numel(), _stream(stream)),
           name)
    return out


def mxattn_prepare(q, k, v, rule="uos", workspace=None, stream=None):
    """Quantize q, k, v (bf16 [B, H, N, d]) into `workspace` (the first half of mxattn_forward)."""
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    if workspace is None:
        workspace = new_workspace(B, H, N, d, q.device)
    qm = _qmax(rule)
    fn, name = (lib().mxattn_prepare, "mxattn_prepare") if qm is None else (lib().mxattn_prepare_qmax,
                                                                             "mxattn_prepare_qmax")
    _check(fn(_cuda(q, "q", torch.bfloat16), _cuda(k, "k", torch.bfloat16), _cuda(v, "v", torch.bfloat16), B, H, N, d,
              _rule(rule) if qm is None else qm, _cuda(workspace, "workspace"), workspace.numel(), _stream(stream)),
           name)
    return workspace


def mxattn_attend(workspace, B, H, N, d, kv_tile=128, pnq=True, rule="uos", softmax_scale=0.0, out=None, stream=None):
    """Attention on a workspace filled by mxattn_prepare (the second half of mxattn_forward)."""
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32, device=workspace.device)
    qm = _qmax(rule)
    fn, name = (lib().mxattn_attend, "mxattn_attend") if qm is None else (lib().mxattn_attend_qmax,
                                                                           "mxattn_attend_qmax")
    _check(fn(B, H, N, d, kv_tile, 1 if pnq else 0, _rule(rule) if qm is None else qm, float(softmax_scale),
              _cuda(out, "out", torch.float32), _cuda(workspace, "workspace"), workspace.numel(), _stream(stream)),
           name)
    return out


def mxattn_forward_quantized(q_codes, q_scales, k_codes, k_scales, vt_codes, vt_scales, B, H, N, d, kv_tile=128,
                             pnq=True, rule="uos", softmax_scale=0.0, out=None, workspace=None, stream=None):
    """Attention on operands already quantized in the public layouts."""
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32, device=q_codes.device)
    if workspace is None:
        workspace = new_workspace(B, H, N, d, q_codes.device)
    _check(lib().mxattn_forward_quantized(
        _cuda(q_codes, "q_codes"), _cuda(q_scales, "q_scales"), _cuda(k_codes, "k_codes"),
        _cuda(k_scales, "k_scales"), _cuda(vt_codes, "vt_codes"), _cuda(vt_scales, "vt_scales"),
        B, H, N, d, kv_tile, 1 if pnq else 0, _rule(rule), float(softmax_scale), _cuda(out, "out", torch.float32),
        _cuda(workspace, "workspace"), workspace.numel(), _stream(stream)), "mxattn_forward_quantized")
    return out


NOALLOC_MAX_WORKSPACE = 16 << 20  # bytes of the library's fixed scratch (include/mxattn.h)


def mxattn_forward_noalloc(q, k, v, kv_tile=128, pnq=True, rule="uos", softmax_scale=0.0, out=None, stream=None):
    """mxattn_forward on the library's fixed scratch: no workspace argument and no
    device allocation inside the call (the output tensor is still the caller's).
    For callers that cannot allocate device memory; shapes whose workspace exceeds
    16 MiB are rejected.  Calls that overlap on the GPU race on the shared scratch."""
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    for name, t in (("k", k), ("v", v), ("out", out)):
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}: all tensors must be on one device")
    # The library's scratch is the one on the current device: make q's device current for the call.
    with torch.cuda.device(q.device):
        s = _stream(torch.cuda.current_stream(q.device) if stream is None else stream)
        _check(lib().mxattn_forward_noalloc(_cuda(q, "q", torch.bfloat16), _cuda(k, "k", torch.bfloat16),
                                            _cuda(v, "v", torch.bfloat16), B, H, N, d, kv_tile, 1 if pnq else 0,
                                            _rule(rule), float(softmax_scale), _cuda(out, "out", torch.float32),
                                            s), "mxattn_forward_noalloc")
    return out


def mxattn_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronize and return the status word of the last forward on `workspace` (0 = ok)."""
    return int(lib().mxattn_workspace_status(_cuda(workspace, "workspace"), _stream(stream)))


def mxattn_wait_selftest(arrive: bool, timeout_us: int, out: torch.Tensor, stream=None) -> None:
    """Launch the bounded-wait self-test; `out` is a device int32[3] tensor that
    holds (status, microseconds waited, flags) once the stream is synchronized."""
    if out.dtype != torch.int32 or out.numel() < 3 or not out.is_contiguous():
        raise MxattnError(1, "out must be a contiguous int32 tensor with 3 elements")
    _check(lib().mxattn_wait_selftest(int(bool(arrive)), int(timeout_us), _cuda(out, "out"), _stream(stream)),
           "mxattn_wait_selftest")


def mxattn_p_selftest(path: int, x: torch.Tensor, qmax: float = 7.25, out=None, stream=None) -> torch.Tensor:
    """The attention kernel's P decisions on inputs x (fp32, numel % 8 == 0):
    E2M1 codes of 2^x (paths 0-2), MXFP4 block exponents (3), NVFP4 block scales (4),
    E2M1 codes of x itself (5)."""
    if out is None:
        out = torch.empty(x.shape, dtype=torch.int32, device=x.device)
    _check(lib().mxattn_p_selftest(int(path), _cuda(x, "x", torch.float32), x.numel(), float(qmax),
                                   _cuda(out, "out", torch.int32), _stream(stream)), "mxattn_p_selftest")
    return out


MXF4_LOOP_FLOP_PER_ITER = 2 * (2 * 128 * 128 * 64)  # two K = 64 MMAs of M = N = 128 per iteration


def mxattn_mxf4_mma_loop(ctas: int, iters: int, status=None, cycles=None, stream=None) -> torch.Tensor:
    """Launch the tensor-core throughput loop (ctas CTAs, 2 * iters block-scaled
    FP4 MMAs each, ctas * iters * MXF4_LOOP_FLOP_PER_ITER flop); returns the
    device status word (0, or MXATTN_ERR_TIMEOUT once the stream has run it).
    `cycles`: optional device int64 [ctas] that receives each CTA's SM clock
    cycles from first issue to last completion."""
    dev = torch.device("cuda", torch.cuda.current_device())
    if status is None:
        status = torch.empty(1, dtype=torch.int32, device=dev)
    cyc = None
    if cycles is not None:
        if cycles.dtype != torch.int64 or cycles.numel() < ctas or not cycles.is_cuda:
            raise MxattnError(1, "cycles must be a CUDA int64 tensor with at least `ctas` elements")
        cyc = _cuda(cycles, "cycles")
    _check(lib().mxattn_mxf4_mma_loop(int(ctas), int(iters), _cuda(status, "status"), cyc, _stream(stream)),
           "mxattn_mxf4_mma_loop")
    return status


def mxattn_status_string(status: int) -> str:
    return status_string(status)


def host_groups(BH: int, chunks: int = 16):
    """Sizes of the (batch, head) groups mxattn_forward_host pipelines by default
    (the library's schedule, restated): `chunks` groups, the first and the last
    of one slice each, the rest as equal as possible."""
    if BH <= 0:
        return []
    n = max(1, min(int(chunks), BH))
    if n < 3 or BH < 3:
        per = -(-BH // n)
        return [min(per, BH - i) for i in range(0, BH, per)]
    mid, k = BH - 2, n - 2
    return [1] + [mid // k + (1 if i < mid % k else 0) for i in range(k)] + [1]


def _group_args(groups, chunks):
    if groups is None:
        return None, int(chunks)
    arr = (ctypes.c_int * len(groups))(*[int(g) for g in groups])
    return arr, len(groups)


def forward_host_workspace_size(B, H, N, d, chunks=16, groups=None) -> int:
    arr, n = _group_args(groups, chunks)
    return int(lib().mxattn_forward_host_workspace_size(B, H, N, d, arr, n))


def attention_from_host(q_host, k_host, v_host, kv_tile=128, pnq=True, rule="uos", softmax_scale=0.0,
                        device_buffers=None, out_host=None, stream=None, chunks=16, groups=None):
    """End-to-end call with host tensors through mxattn_forward_host: q, k, v
    (pinned host bf16 [B, H, N, d]) to the device, the attention, O back into
    `out_host` (pinned fp32), pipelined over (batch, head) groups inside the
    library (`groups`: their sizes, summing to B*H; default: `chunks` groups).
    The work is ordered on `stream` (default: the current stream).
    `device_buffers` = (q, k, v, out, workspace) device tensors to reuse; the
    workspace needs forward_host_workspace_size(...) bytes."""
    B, H, N, d = q_host.shape
    BH = B * H
    dev = torch.device("cuda", torch.cuda.current_device())
    if device_buffers is None:
        device_buffers = (torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev),
                          torch.empty((B, H, N, d), dtype=torch.float32, device=dev), None)
    qd, kd, vd, od, ws = device_buffers
    if out_host is None:
        out_host = torch.empty((B, H, N, d), dtype=torch.float32, pin_memory=True)
    if groups is not None:
        sizes = [int(g) for g in groups]
        if BH and (sum(sizes) != BH or min(sizes) < 1):
            raise ValueError(f"groups {sizes} must be positive and sum to B*H = {BH}")
    arr, n = _group_args(groups, chunks)
    if ws is None:
        need = int(lib().mxattn_forward_host_workspace_size(B, H, N, d, arr, n))
        if need == 0:
            raise MxattnError(1, "mxattn_forward_host_workspace_size")
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    for name, t in (("q", q_host), ("k", k_host), ("v", v_host), ("out", out_host)):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    if q_host.dtype != torch.bfloat16 or out_host.dtype != torch.float32:
        raise ValueError("q, k, v must be bfloat16 and out float32")
    hp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    _check(lib().mxattn_forward_host(hp(q_host), hp(k_host), hp(v_host), B, H, N, d, kv_tile, 1 if pnq else 0,
                                     _rule(rule), float(softmax_scale), hp(out_host), _cuda(qd, "q_dev"),
                                     _cuda(kd, "k_dev"), _cuda(vd, "v_dev"), _cuda(od, "o_dev", torch.float32),
                                     _cuda(ws, "workspace"), ws.numel(), arr, n, _stream(stream)),
           "mxattn_forward_host")
    return out_host


# ---------------------------------------------------------------- NVFP4 comparison variant

def mxattn_nvfp4_quantize(x: torch.Tensor, codes=None, scales=None, gs=None, stream=None):
    """bf16 [..., cols] (cols % 16 == 0) -> (codes u8 [..., cols/2], E4M3 scales u8 [..., cols/16],
    gs fp32 [2] = (amax, g)), one second-level scale g for the whole tensor."""
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (cols // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (cols // 16,), dtype=torch.uint8, device=x.device)
    if gs is None:
        gs = torch.empty(2, dtype=torch.float32, device=x.device)
    _check(lib().mxattn_nvfp4_quantize(_cuda(x, "x", torch.bfloat16), rows, cols, _cuda(codes, "codes"),
                                       _cuda(scales, "scales"), _cuda(gs, "gs", torch.float32), _stream(stream)),
           "mxattn_nvfp4_quantize")
    return codes, scales, gs


def nvfp4_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(lib().mxattn_nvfp4_workspace_size(B, H, N, d))


def nvfp4_workspace_layout(B: int, H: int, N: int, d: int) -> dict:
    """Byte offsets of the NVFP4 workspace regions (as documented in include/mxattn.h)."""
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    BH, G, npad = B * H, (N + 127) // 128, (N + 31) // 32 * 32
    off, out = 0, {}
    for name, size in (("status", 256), ("q_codes", BH * N * d // 2), ("k_codes", BH * N * d // 2),
                       ("vt_codes", BH * d * npad // 2), ("q_sf", BH * G * (d // 64) * 512),
                       ("k_sf", BH * G * (d // 64) * 512), ("vt_sf", BH * G * 1024), ("amax", 3 * BH * 4),
                       ("g", 3 * BH * 4)):
        out[name] = (off, size)
        off = a(off + size)
    out["total"] = off
    return out


def new_nvfp4_workspace(B, H, N, d, device="cuda") -> torch.Tensor:
    n = nvfp4_workspace_size(B, H, N, d)
    if n == 0:
        raise MxattnError(1, "mxattn_nvfp4_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def mxattn_nvfp4_forward(q, k, v, kv_tile=128, pnq=True, softmax_scale=0.0, out=None, workspace=None, stream=None):
    """NVFP4 attention: q, k, v bf16 [B, H, N, d] -> O fp32 [B, H, N, d]."""
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_nvfp4_workspace(B, H, N, d, q.device)
    _check(lib().mxattn_nvfp4_forward(_cuda(q, "q", torch.bfloat16), _cuda(k, "k", torch.bfloat16),
                                      _cuda(v, "v", torch.bfloat16), B, H, N, d, kv_tile, 1 if pnq else 0,
                                      float(softmax_scale), _cuda(out, "out", torch.float32),
                                      _cuda(workspace, "workspace"), workspace.numel(), _stream(stream)),
           "mxattn_nvfp4_forward")
    return out


def mxattn_nvfp4_prepare(q, k, v, workspace=None, stream=None):
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, H, N, d]")
    if workspace is None:
        workspace = new_nvfp4_workspace(B, H, N, d, q.device)
    _check(lib().mxattn_nvfp4_prepare(_cuda(q, "q", torch.bfloat16), _cuda(k, "k", torch.bfloat16),
                                      _cuda(v, "v", torch.bfloat16), B, H, N, d, _cuda(workspace, "workspace"),
                                      workspace.numel(), _stream(stream)), "mxattn_nvfp4_prepare")
    return workspace


def mxattn_nvfp4_attend(workspace, B, H, N, d, kv_tile=128, pnq=True, softmax_scale=0.0, out=None, stream=None):
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32, device=workspace.device)
    _check(lib().mxattn_nvfp4_attend(B, H, N, d, kv_tile, 1 if pnq else 0, float(softmax_scale),
                                     _cuda(out, "out", torch.float32), _cuda(workspace, "workspace"),
                                     workspace.numel(), _stream(stream)), "mxattn_nvfp4_attend")
    return out
