"""Randomized parity sweep of both attention paths (MXFP4 with UOS / OCP /
other scale boundaries, and the NVFP4 comparison variant) against the CPU
oracle, over seeded random shapes, tiles, PNQ settings, softmax scales and
input distributions.

Criteria (MXAttention abstract, "MXAttention: Data-Free Optimal Scaling and
Pre-Normalization Quantization for MXFP4 Attention"; the target's tolerance
for O is rel-Frobenius <= 1e-3 and max-abs <= 2e-2):
  - Q, K, V^T codes and scales: bit for bit;
  - O: max-abs <= 2e-2 and rel-Frobenius <= 1e-3 over every checked row of
    every case, no row excluded.
As a printed diagnostic only, each case reports how many rows a P decision
flip touched.  The kernel decides P's codes in fp32 and the oracle in fp64,
so an exponential within fp32 rounding of a rounding point may round the
other way; that moves one weight of one row by one E2M1 step, so that row's
error jumps from about 1e-7 to as much as a few percent.  A row counts as
touched above 1e-5 relative error; without PNQ the row sum adds unquantized
fp32 exponentials whose exponents carry the fp32 rounding of m * kq, so rows
with large scores (|m kq| in the hundreds) differ from the fp64 oracle by a
common factor up to ln 2 * ulp(|m kq|), which is added to that threshold.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200 import workloads as wl

from test_attention_gpu import check_codes, sampled_rows
from test_nvfp4_gpu import check_workspace
from test_quantize_gpu import _dev

pytestmark = pytest.mark.gpu

CASES = 24


def _inputs(rng, B, H, N, d):
    kind = rng.choice(["gaussian", "student_t", "outlier", "wide"])
    seed = int(rng.integers(1 << 30))
    if kind == "gaussian":
        Q, K, V = wl.gaussian_qkv(B, H, N, d, seed=seed)
    elif kind == "student_t":
        Q, K, V = wl.student_t_qkv(B, H, N, d, seed=seed)
    elif kind == "outlier":
        Q, K, V = wl.outlier_qkv(B, H, N, d, seed=seed, factor=float(rng.uniform(4, 12)))
    else:  # magnitudes spread over many binades, per head and per row
        r = np.random.default_rng(seed)
        out = []
        for _ in range(3):
            x = r.standard_normal((B, H, N, d)).astype(np.float32)
            x *= np.exp2(r.uniform(-6, 6, (B, H, 1, 1)) + r.uniform(-2, 2, (B, H, N, 1))).astype(np.float32)
            out.append(wl.f32_to_bf16_bits(x))
        Q, K, V = out
    return kind, Q, K, V


def _exponent_bias_bound(Q, K, rows, scale, rule=None):
    """Per row, an upper bound on the relative error that the fp32 exponent bias
    puts into a row sum of unquantized exponentials (PNQ off).  The kernel forms
    each exponent as fma(s, kq, -(m kq + e)) with m kq rounded to fp32, so every
    exponential of row i (the row maximum's included) carries a relative error
    up to ln 2 * ulp(|m_i kq| + 128); the sum inherits it.  With PNQ the row sum
    adds the quantized values instead, which this does not move.  m_i is the
    row's score maximum over the dequantized operands (oracle quantizers; rule
    None: NVFP4)."""
    B, H, N, d = Q.shape
    kq = (scale if scale > 0 else 1.0 / np.sqrt(d)) / np.log(2.0)
    out = np.empty((B, H, len(rows)))
    for b in range(B):
        for h in range(H):
            if rule is None:
                gq, gk = (oracle.nvfp4_head_globals(X[b:b + 1, h:h + 1])[0, 0] for X in (Q, K))
                qd = oracle.nvfp4_dequantize_rows(*oracle.nvfp4_quantize_rows(Q[b, h][rows], gq), gq)
                kd = oracle.nvfp4_dequantize_rows(*oracle.nvfp4_quantize_rows(K[b, h], gk), gk)
            else:
                qd = oracle.dequantize_rows(*oracle.quantize_rows(Q[b, h][rows], rule))
                kd = oracle.dequantize_rows(*oracle.quantize_rows(K[b, h], rule))
            m = (qd.reshape(len(rows), d) @ kd.reshape(N, d).T).max(axis=1)
            out[b, h] = 2.0 * np.log(2.0) * (np.abs(m) * kq + 130.0) * 2.0 ** -23
    return out


def _check_o(O, R, what, row_bound=None):
    """max-abs <= 2e-2 and rel-Frobenius <= 1e-3 over all rows; returns the number of
    rows a P decision flip touched (relative error above 1e-5, plus row_bound, the fp32
    exponent-bias bound of PNQ-off rows) as a diagnostic."""
    assert np.all(np.isfinite(O)), what
    mabs = float(np.max(np.abs(O - R)))
    rel = float(np.linalg.norm(O - R) / np.linalg.norm(R))
    rows = np.linalg.norm(O - R, axis=-1) / np.maximum(np.linalg.norm(R, axis=-1), 1e-30)
    touched = rows > 1e-5 + (0.0 if row_bound is None else row_bound)
    assert mabs <= 2e-2, f"{what}: max-abs {mabs:.3e} ({touched.sum()} rows touched by P flips)"
    assert rel <= 1e-3, f"{what}: rel-Frobenius {rel:.3e} over all rows ({touched.sum()} rows touched by P flips)"
    return int(touched.sum()), rel, mabs


@pytest.mark.parametrize("case", range(CASES))
def test_random_configuration(case):
    rng = np.random.default_rng(1000 + case)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    N = int(rng.choice([int(rng.integers(1, 200)), int(rng.integers(200, 1500))]))
    d, T = int(rng.choice([64, 128])), int(rng.choice([64, 128]))
    pnq = bool(rng.integers(2))
    scale = float(np.float32(rng.choice([0.0, rng.uniform(0.02, 0.3)])))  # the kernel takes an fp32 scale
    kind, Q, K, V = _inputs(rng, B, H, N, d)
    what = f"case {case}: B={B} H={H} N={N} d={d} T={T} pnq={pnq} scale={scale:.3f} {kind}"
    if case % 3 == 2:  # the NVFP4 comparison variant
        ws = mx.new_nvfp4_workspace(B, H, N, d)
        O = mx.mxattn_nvfp4_forward(_dev(Q), _dev(K), _dev(V), T, pnq, scale, workspace=ws)
        assert mx.mxattn_workspace_status(ws) == 0
        R = oracle.nvfp4_attention(Q, K, V, T, pnq=pnq, scale=scale if scale > 0 else None)
        check_workspace(ws, Q, K, V)
        what += " nvfp4"
    else:
        rule = [["uos", "ocp"][case % 2], float(rng.choice([4.5, 5.0, 6.0, 6.5, 7.0, 7.5, 7.875]))][(case // 3) % 2]
        ws = mx.new_workspace(B, H, N, d)
        O = mx.mxattn_forward(_dev(Q), _dev(K), _dev(V), T, pnq, rule, scale, workspace=ws)
        assert mx.mxattn_workspace_status(ws) == 0
        R = oracle.attention(Q, K, V, T, rule=rule, pnq=pnq, scale=scale if scale > 0 else None)
        check_codes(ws, Q, K, V, rule)
        what += f" rule={rule}"
    bound = None if pnq else _exponent_bias_bound(Q, K, np.arange(N), scale, None if case % 3 == 2 else rule)
    touched, rel, mabs = _check_o(O.cpu().numpy().astype(np.float64), R, what, bound)
    print(f"[fuzz] {what}: rows touched {touched}, rel {rel:.2e}, max-abs {mabs:.2e}")


LONG_CASES = 8


@pytest.mark.parametrize("case", range(LONG_CASES))
def test_random_long_configuration(case):
    """The same criteria on long key loops (N in [2000, 8000): 16 to 125 key
    tiles, with many running-max moves and O rescales), O checked on 256 seeded
    rows plus the first and last rows and the tile edges, for every head."""
    rng = np.random.default_rng(5000 + case)
    B, H = 1, int(rng.integers(1, 3))
    N = int(rng.integers(2000, 8000))
    d, T = int(rng.choice([64, 128])), int(rng.choice([64, 128]))
    pnq = bool(rng.integers(2))
    scale = float(np.float32(rng.choice([0.0, rng.uniform(0.02, 0.3)])))
    kind, Q, K, V = _inputs(rng, B, H, N, d)
    rows = sampled_rows(N, 256, 77 + case)
    what = f"long case {case}: H={H} N={N} d={d} T={T} pnq={pnq} scale={scale:.3f} {kind}"
    sc = scale if scale > 0 else None
    if case % 4 == 3:
        ws = mx.new_nvfp4_workspace(B, H, N, d)
        O = mx.mxattn_nvfp4_forward(_dev(Q), _dev(K), _dev(V), T, pnq, scale, workspace=ws)
        assert mx.mxattn_workspace_status(ws) == 0
        R = oracle.nvfp4_attention(Q, K, V, T, pnq=pnq, scale=sc, rows=rows)
        check_workspace(ws, Q, K, V)
        what += " nvfp4"
    else:
        rule = ["uos", "ocp", float(rng.choice([5.0, 6.5, 7.5]))][case % 3]
        ws = mx.new_workspace(B, H, N, d)
        O = mx.mxattn_forward(_dev(Q), _dev(K), _dev(V), T, pnq, rule, scale, workspace=ws)
        assert mx.mxattn_workspace_status(ws) == 0
        R = oracle.attention(Q, K, V, T, rule=rule, pnq=pnq, scale=sc, rows=rows)
        check_codes(ws, Q, K, V, rule)
        what += f" rule={rule}"
    got = O.cpu().numpy().astype(np.float64)[:, :, rows]
    bound = None if pnq else _exponent_bias_bound(Q, K, rows, scale, None if case % 4 == 3 else rule)
    touched, rel, mabs = _check_o(got, R, what, bound)
    print(f"[fuzz-long] {what}: rows touched {touched} of {got.shape[1] * got.shape[2]}, rel {rel:.2e}, "
          f"max-abs {mabs:.2e}")
