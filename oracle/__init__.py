"""CPU oracle for MXFP4 attention with UOS and PNQ (fp64, plain C loops).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package.  It shares no code with the CUDA library; both take
their inputs from ``mxfp4_microscaled_quantization_b200.workloads``.

What each function computes, and the reading behind it, is documented beside
the C code in ``oracle.c`` (source: the MXAttention abstract, "MXAttention:
Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
Attention").  Every function here is pinned by the ``-m "not gpu"`` tests
(E2M1 grid and brute-force rounding, the OCP and UOS scale invariants,
equivariance, exact online softmax, PNQ normalization, hand-derived golden
cases, and two-key-tile cases of the quantized loop with values derived by
hand, which fail if P is quantized against the tile-local or the final row
maximum; for the NVFP4 comparison variant, torch's float8_e4m3fn conversion,
brute-force element rounding, equivariance, special cases and the same
two-tile cases); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

RULES = {"ocp": 0, "uos": 1, "none": 2}
RULE_QMAX = 3  # boundary rule with a caller-chosen Qmax in (4, 8)
UOS_QMAX = 7.25


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (fp64, no fast-math, no FMA contraction, OpenMP over rows)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(_LIB_PATH)
    return _lib


def load(path: str) -> ctypes.CDLL:
    """Open a compiled oracle library at `path` and declare its signatures."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    L.oracle_e2m1_encode_batch.argtypes = [P, i64, P]
    L.oracle_scale_exponent_batch.argtypes = [P, i64, ctypes.c_int, P]
    L.oracle_scale_exponent_q_batch.argtypes = [P, i64, ctypes.c_int, ctypes.c_double, P]
    L.oracle_quantize_rows_q.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_double, P, P]
    L.oracle_quantize_cols_q.argtypes = [P, i64, i64, i64, ctypes.c_int, ctypes.c_double, P, P]
    L.oracle_attention_head_q.argtypes = [P, P, P, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_int, ctypes.c_double, P, i64, P, ctypes.c_int]
    L.oracle_attention_head_q.restype = ctypes.c_int
    L.oracle_quantize_rows.argtypes = [P, i64, i64, ctypes.c_int, P, P]
    L.oracle_quantize_cols.argtypes = [P, i64, i64, i64, ctypes.c_int, P, P]
    L.oracle_dequantize_rows.argtypes = [P, P, i64, i64, P]
    L.oracle_attention_head.argtypes = [P, P, P, i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, P, i64, P, ctypes.c_int]
    L.oracle_attention_head.restype = ctypes.c_int
    L.oracle_max_threads.restype = ctypes.c_int
    L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_decode.restype = ctypes.c_double
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = ctypes.c_double
    L.oracle_e4m3_encode_batch.argtypes = [P, i64, P]
    L.oracle_nvfp4_global.argtypes = [ctypes.c_double]
    L.oracle_nvfp4_global.restype = ctypes.c_float
    L.oracle_bf16_amax.argtypes = [P, i64]
    L.oracle_bf16_amax.restype = ctypes.c_double
    L.oracle_nvfp4_quantize_rows.argtypes = [P, i64, i64, ctypes.c_float, P, P]
    L.oracle_nvfp4_quantize_cols.argtypes = [P, i64, i64, i64, P, P, P]
    L.oracle_nvfp4_dequantize_rows.argtypes = [P, P, i64, i64, ctypes.c_float, P]
    L.oracle_nvfp4_attention_head.argtypes = [P, P, P, i64, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_double, P, i64, P, ctypes.c_int]
    L.oracle_nvfp4_attention_head.restype = ctypes.c_int
    return L


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _rule(r):
    """Rule name ("ocp", "uos", "none") or a scale boundary Qmax -> (rule code, Qmax).

    A numeric Qmax in (4, 8) selects the boundary rule "smallest e with
    amax <= Qmax * 2^e"; Qmax = 8 selects OCP, the limit of that rule as Qmax
    approaches 8 from below."""
    if isinstance(r, str):
        return RULES[r], UOS_QMAX
    q = float(r)
    if q == 8.0:
        return RULES["ocp"], q
    if not 4.0 < q < 8.0:
        raise ValueError(f"Qmax must lie in (4, 8], got {q}")
    return RULE_QMAX, q


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def e2m1_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    return np.array([lib().oracle_e2m1_decode(int(c)) for c in codes.ravel()]).reshape(codes.shape)


def e2m1_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e2m1_encode_batch(_ptr(v), v.size, _ptr(out))
    return out


def scale_exponent(amax, rule) -> np.ndarray:
    a = np.ascontiguousarray(amax, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.int32)
    code, q = _rule(rule)
    lib().oracle_scale_exponent_q_batch(_ptr(a), a.size, code, q, _ptr(out))
    return out


def quantize_rows(x_bits: np.ndarray, rule):
    """bf16 bits [rows, cols] -> (codes uint8 [rows, cols/2], scales uint8 [rows, cols/32])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    cols = x.shape[-1]
    assert cols % 32 == 0
    rows = x.size // cols
    codes = np.empty(x.shape[:-1] + (cols // 2,), dtype=np.uint8)
    scales = np.empty(x.shape[:-1] + (cols // 32,), dtype=np.uint8)
    code, q = _rule(rule)
    lib().oracle_quantize_rows_q(_ptr(x), rows, cols, code, q, _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_cols(v_bits: np.ndarray, rule):
    """V bf16 bits [..., N, d] -> V^T (codes [..., d, Npad/2], scales [..., d, Npad/32])."""
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    N, d = v.shape[-2:]
    BH = v.size // (N * d)
    npad = (N + 31) // 32 * 32
    lead = v.shape[:-2]
    codes = np.empty(lead + (d, npad // 2), dtype=np.uint8)
    scales = np.empty(lead + (d, npad // 32), dtype=np.uint8)
    code, q = _rule(rule)
    lib().oracle_quantize_cols_q(_ptr(v), BH, N, d, code, q, _ptr(codes), _ptr(scales))
    return codes, scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    cols = codes.shape[-1] * 2
    rows = codes.size * 2 // cols
    out = np.empty(codes.shape[:-1] + (cols,), dtype=np.float64)
    lib().oracle_dequantize_rows(_ptr(codes), _ptr(scales), rows, cols, _ptr(out))
    return out


def attention(Q, K, V, kv_tile, rule="uos", pnq=True, p_rule=None, scale=None, rows=None, nthreads=0):
    """MXFP4 attention forward on the CPU in fp64.

    Q, K, V: bf16 bits [B, H, N, d].  `rule` quantizes Q, K, V (and P unless
    `p_rule` says otherwise); "none" disables quantization; a number is a
    scale boundary Qmax in (4, 8] (see `_rule`).  A numeric `rule` and a
    numeric `p_rule` must name the same Qmax.  `rows`: None for
    all rows, else an int array of query rows (the same rows for every head)
    or a list with one array per (b, h).  Returns fp64 [B, H, R, d].
    """
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    K = np.ascontiguousarray(K, dtype=np.uint16)
    V = np.ascontiguousarray(V, dtype=np.uint16)
    B, H, N, d = Q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    in_rule, q_in = _rule(rule)
    pr, q_p = (in_rule, q_in) if p_rule is None else _rule(p_rule)
    qmax = q_in if in_rule == RULE_QMAX else q_p
    if in_rule == RULE_QMAX and pr == RULE_QMAX and q_in != q_p:
        raise ValueError("rule and p_rule must name the same Qmax")
    per_head_rows = []
    for bh in range(B * H):
        if rows is None:
            r = np.arange(N, dtype=np.int64)
        elif isinstance(rows, (list, tuple)):
            r = np.asarray(rows[bh], dtype=np.int64)
        else:
            r = np.asarray(rows, dtype=np.int64)
        per_head_rows.append(np.ascontiguousarray(r))
    R = len(per_head_rows[0])
    assert all(len(r) == R for r in per_head_rows)
    out = np.empty((B, H, R, d), dtype=np.float64)
    Qf = Q.reshape(B * H, N, d)
    Kf = K.reshape(B * H, N, d)
    Vf = V.reshape(B * H, N, d)
    ov = out.reshape(B * H, R, d)
    for bh in range(B * H):
        o = np.empty((R, d), dtype=np.float64)
        st = lib().oracle_attention_head_q(_ptr(Qf[bh]), _ptr(Kf[bh]), _ptr(Vf[bh]), N, d, kv_tile, in_rule, pr,
                                           float(qmax), 1 if pnq else 0, float(scale), _ptr(per_head_rows[bh]), R,
                                           _ptr(o), int(nthreads))
        if st != 0:
            raise RuntimeError(f"oracle_attention_head failed with status {st}")
        ov[bh] = o
    return out


# ---------------------------------------------------------------- NVFP4 comparison variant
# Definitions and readings beside the C code (oracle.c, "NVFP4 comparison variant").

def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    return np.array([lib().oracle_e4m3_decode(int(c)) for c in codes.ravel()]).reshape(codes.shape)


def e4m3_encode(v) -> np.ndarray:
    """|v| -> E4M3 code, round to nearest even, saturating at 448."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_batch(_ptr(v), v.size, _ptr(out))
    return out


def nvfp4_global(amax) -> np.float32:
    """Second-level scale g = 448 / amax (fp32) of a slice with absolute maximum amax."""
    return np.float32(lib().oracle_nvfp4_global(float(amax)))


def nvfp4_head_globals(x_bits: np.ndarray) -> np.ndarray:
    """bf16 bits [B, H, N, d] -> g per (batch, head), float32 [B, H]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    B, H = x.shape[:2]
    flat = x.reshape(B * H, -1)
    g = [nvfp4_global(lib().oracle_bf16_amax(_ptr(np.ascontiguousarray(flat[i])), flat.shape[1]))
         for i in range(B * H)]
    return np.array(g, dtype=np.float32).reshape(B, H)


def nvfp4_quantize_rows(x_bits: np.ndarray, g):
    """bf16 bits [rows, cols] (cols % 16 == 0), one scale g -> (codes [rows, cols/2], E4M3 scales [rows, cols/16])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    cols = x.shape[-1]
    assert cols % 16 == 0
    rows = x.size // cols
    codes = np.empty(x.shape[:-1] + (cols // 2,), dtype=np.uint8)
    scales = np.empty(x.shape[:-1] + (cols // 16,), dtype=np.uint8)
    lib().oracle_nvfp4_quantize_rows(_ptr(x), rows, cols, float(g), _ptr(codes), _ptr(scales))
    return codes, scales


def nvfp4_quantize_cols(v_bits: np.ndarray, g):
    """V bf16 bits [BH..., N, d], g one scale per (b, h) -> V^T (codes [..., d, Npad/2], scales [..., d, Npad/16])."""
    v = np.ascontiguousarray(v_bits, dtype=np.uint16)
    N, d = v.shape[-2:]
    BH = v.size // (N * d)
    npad = (N + 31) // 32 * 32
    lead = v.shape[:-2]
    gg = np.ascontiguousarray(np.broadcast_to(np.asarray(g, dtype=np.float32).ravel(), (BH,)))
    codes = np.empty(lead + (d, npad // 2), dtype=np.uint8)
    scales = np.empty(lead + (d, npad // 16), dtype=np.uint8)
    lib().oracle_nvfp4_quantize_cols(_ptr(v), BH, N, d, _ptr(gg), _ptr(codes), _ptr(scales))
    return codes, scales


def nvfp4_dequantize_rows(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    cols = codes.shape[-1] * 2
    rows = codes.size * 2 // cols
    out = np.empty(codes.shape[:-1] + (cols,), dtype=np.float64)
    lib().oracle_nvfp4_dequantize_rows(_ptr(codes), _ptr(scales), rows, cols, float(g), _ptr(out))
    return out


def nvfp4_attention(Q, K, V, kv_tile, pnq=True, quant=True, p_quant=True, scale=None, rows=None, nthreads=0):
    """NVFP4 attention forward on the CPU (fp64 loop, fp32 scale arithmetic).

    Q, K, V: bf16 bits [B, H, N, d].  quant=False keeps every operand exact;
    p_quant=False keeps only P exact.  rows as in `attention`.  Returns fp64 [B, H, R, d].
    """
    Q = np.ascontiguousarray(Q, dtype=np.uint16)
    K = np.ascontiguousarray(K, dtype=np.uint16)
    V = np.ascontiguousarray(V, dtype=np.uint16)
    B, H, N, d = Q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    per_head_rows = []
    for bh in range(B * H):
        if rows is None:
            r = np.arange(N, dtype=np.int64)
        elif isinstance(rows, (list, tuple)):
            r = np.asarray(rows[bh], dtype=np.int64)
        else:
            r = np.asarray(rows, dtype=np.int64)
        per_head_rows.append(np.ascontiguousarray(r))
    R = len(per_head_rows[0])
    out = np.empty((B, H, R, d), dtype=np.float64)
    Qf, Kf, Vf = (a.reshape(B * H, N, d) for a in (Q, K, V))
    ov = out.reshape(B * H, R, d)
    for bh in range(B * H):
        o = np.empty((R, d), dtype=np.float64)
        st = lib().oracle_nvfp4_attention_head(_ptr(Qf[bh]), _ptr(Kf[bh]), _ptr(Vf[bh]), N, d, kv_tile,
                                               1 if quant else 0, 1 if p_quant else 0, 1 if pnq else 0,
                                               float(scale), _ptr(per_head_rows[bh]), R, _ptr(o), int(nthreads))
        if st != 0:
            raise RuntimeError(f"oracle_nvfp4_attention_head failed with status {st}")
        ov[bh] = o
    return out
