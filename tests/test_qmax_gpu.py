"""Parity of the scale-boundary (Qmax) entry points with the CPU oracle.

The MXAttention abstract ("MXAttention: Data-Free Optimal Scaling and
Pre-Normalization Quantization for MXFP4 Attention") names the UOS scaling
boundary Qmax and picks 7.25; the *_qmax entry points take any boundary in
(4, 8] for the same rule (Qmax = 8 is the OCP rule).  Codes and scales must
match the oracle bit for bit at every boundary; O within the attention
tolerance (relative Frobenius <= 1e-3, max-abs <= 2e-2).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200 import workloads as wl

from test_attention_gpu import assert_close, check_codes, run_forward
from test_quantize_gpu import _dev, _exponent_sweep_blocks, _finite_patterns

pytestmark = pytest.mark.gpu

# 7.25 (UOS) and 8 (OCP) included; all exactly representable in fp32.
QMAX = [4.5, 5.0, 6.0, 6.5, 7.0, 7.25, 7.5, 7.875, 8.0]


def _gpu_rows(bits, qmax):
    c, s = mx.mxattn_quantize(_dev(bits), qmax)
    torch.cuda.synchronize()
    return c.cpu().numpy(), s.cpu().numpy()


def _every_block_maximum():
    amax = np.arange(1, 0x7F80, dtype=np.uint16)
    rng = np.random.default_rng(21)
    x = rng.integers(0, 1 << 15, size=(len(amax), 32), dtype=np.uint16)
    x = np.minimum(x, amax[:, None])
    x[:, 0] = amax
    x |= rng.integers(0, 2, size=x.shape, dtype=np.uint16) << 15
    return x[: len(x) // 4 * 4].reshape(-1, 128)


@pytest.mark.parametrize("qmax", QMAX)
def test_quantize_qmax_every_block_maximum(qmax):
    x = _every_block_maximum()
    gc, gs = _gpu_rows(x, qmax)
    oc, os_ = oracle.quantize_rows(x, qmax)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, oc)


@pytest.mark.parametrize("qmax", [5.0, 6.0, 7.5])
def test_quantize_qmax_every_exponent_tie_and_pattern(qmax):
    x = _exponent_sweep_blocks()
    gc, gs = _gpu_rows(x, qmax)
    oc, os_ = oracle.quantize_rows(x, qmax)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, oc)
    pats = _finite_patterns()
    x = np.random.default_rng(22).permutation(pats)
    x = x[: len(x) // 4096 * 4096].reshape(-1, 4096)
    gc, gs = _gpu_rows(x, qmax)
    oc, os_ = oracle.quantize_rows(x, qmax)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, oc)


def test_named_rules_are_their_boundaries():
    """mxattn_quantize(rule) == mxattn_quantize_qmax at 7.25 (UOS) and 8 (OCP), bit for bit."""
    x = _every_block_maximum()
    for rule, q in (("uos", 7.25), ("ocp", 8.0)):
        a = _gpu_rows(x, rule)
        b = _gpu_rows(x, q)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_qmax_outside_the_family_is_rejected():
    x = _dev(np.zeros((4, 64), dtype=np.uint16))
    for q in (4.0, 3.5, 8.25, float("nan")):
        with pytest.raises(mx.MxattnError):
            mx.mxattn_quantize(x, q)


@pytest.mark.parametrize("qmax", [6.0, 7.5])
@pytest.mark.parametrize("pnq", [True, False])
def test_attention_qmax_tiny(qmax, pnq):
    w = wl.WORKLOADS["tiny"]
    Q, K, V = wl.make_qkv(w, seed=0)
    O, ws = run_forward(Q, K, V, w.kv_tile, pnq, qmax)
    R = oracle.attention(Q, K, V, w.kv_tile, rule=qmax, pnq=pnq)
    assert_close(O, R, f"tiny qmax={qmax} pnq={pnq}")
    check_codes(ws, Q, K, V, qmax)


@pytest.mark.parametrize("qmax", [5.0, 6.5])
def test_attention_qmax_ragged(qmax):
    for N, d, T in ((257, 128, 128), (100, 64, 64)):
        Q, K, V = wl.gaussian_qkv(1, 2, N, d, seed=N + d)
        Q = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(Q) * np.float32(2.0))
        O, ws = run_forward(Q, K, V, T, True, qmax)
        R = oracle.attention(Q, K, V, T, rule=qmax, pnq=True)
        assert_close(O, R, f"N={N} d={d} T={T} qmax={qmax}")
        check_codes(ws, Q, K, V, qmax)


def test_attention_named_rule_equals_its_boundary():
    w = wl.WORKLOADS["tiny"]
    Q, K, V = wl.make_qkv(w, seed=5)
    for rule, q in (("uos", 7.25), ("ocp", 8.0)):
        a, _ = run_forward(Q, K, V, w.kv_tile, True, rule)
        b, _ = run_forward(Q, K, V, w.kv_tile, True, q)
        np.testing.assert_array_equal(a, b)
