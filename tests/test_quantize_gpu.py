"""Bit-exact parity of the CUDA quantize kernels with the CPU oracle (E2M1
codes and E8M0 scales under the OCP and UOS rules; MXAttention abstract,
"MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for
MXFP4 Attention")."""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

RULES = ("ocp", "uos")


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _gpu_rows(bits, rule):
    c, s = mx.mxattn_quantize(_dev(bits), rule)
    torch.cuda.synchronize()
    return c.cpu().numpy(), s.cpu().numpy()


def _finite_patterns():
    b = np.arange(1 << 16, dtype=np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


def _exponent_sweep_blocks():
    """For every block exponent reachable from bf16 maxima: blocks led by +-6*2^e
    (exponent e under both rules) holding the E2M1 rounding ties
    {0.25,0.75,1.25,1.75,2.5,3.5,5}*2^e, their bf16 neighbours, and every
    mantissa of the binades around 2^e with both signs."""
    rows = []
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 0.5, 1.0])
    mant = np.arange(128, dtype=np.uint16)
    for e in range(-134, 126):
        lead = np.float32(np.ldexp(6.0, e))
        vals = [np.ldexp(ties, e).astype(np.float32)]
        base = wl.f32_to_bf16_bits(vals[0])
        for exp_field in range(max(0, e + 127 - 4), min(254, e + 127 + 3) + 1):
            vals.append(wl.bf16_bits_to_f32((exp_field << 7) | mant))
        v = np.concatenate(vals)
        bits = np.concatenate([base, base + 1, base - 1, wl.f32_to_bf16_bits(v)])
        bits = np.concatenate([bits, bits | 0x8000])
        bits = bits[(bits & 0x7FFF) <= wl.f32_to_bf16_bits(np.array([lead]))[0]]
        nblk = (len(bits) + 30) // 31
        body = np.zeros(nblk * 31, dtype=np.uint16)
        body[: len(bits)] = bits
        blk = np.empty((nblk, 32), dtype=np.uint16)
        blk[:, 0] = wl.f32_to_bf16_bits(np.array([lead]))[0] | (np.arange(nblk) % 2 * 0x8000).astype(np.uint16)
        blk[:, 1:] = body.reshape(nblk, 31)
        rows.append(blk)
    return np.concatenate(rows).reshape(-1, 32)


@pytest.mark.parametrize("rule", RULES)
def test_quantize_all_bf16_patterns_random_blocks(rule):
    pats = _finite_patterns()
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.permutation(pats) for _ in range(4)])
    x = x[: len(x) // 4096 * 4096].reshape(-1, 4096)
    gc, gs = _gpu_rows(x, rule)
    oc, os_ = oracle.quantize_rows(x, rule)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, oc)


@pytest.mark.parametrize("rule", RULES)
def test_quantize_every_exponent_and_tie(rule):
    x = _exponent_sweep_blocks()
    gc, gs = _gpu_rows(x, rule)
    oc, os_ = oracle.quantize_rows(x, rule)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, oc)


@pytest.mark.parametrize("rule", RULES)
def test_quantize_every_block_maximum(rule):
    """One block per positive finite bf16 maximum (32640 blocks): the scale rule on every amax."""
    amax = np.arange(1, 0x7F80, dtype=np.uint16)
    rng = np.random.default_rng(1)
    x = rng.integers(0, 1 << 15, size=(len(amax), 32), dtype=np.uint16)
    x = np.minimum(x, amax[:, None])  # |x| <= amax as bit patterns
    x[:, 0] = amax
    x |= (rng.integers(0, 2, size=x.shape, dtype=np.uint16) << 15)
    x = x[: len(x) // 4 * 4].reshape(-1, 128)
    gc, gs = _gpu_rows(x, rule)
    oc, os_ = oracle.quantize_rows(x, rule)
    np.testing.assert_array_equal(gs, os_)
    np.testing.assert_array_equal(gc, oc)


def test_negative_zero_and_sign_of_underflow():
    x = np.zeros((1, 32), dtype=np.uint16)
    x[0, 0] = 0x40C0  # 6.0 -> e = 0
    x[0, 1] = 0x8000  # -0.0
    x[0, 2] = 0xBD80  # -0.0625 -> rounds to -0
    x[0, 3] = 0x3D80  # +0.0625 -> +0
    for rule in RULES:
        gc, gs = _gpu_rows(x, rule)
        assert gs[0, 0] == 127
        assert gc[0, 0] == 0x7 | (0x8 << 4)
        assert gc[0, 1] == 0x8 | (0x0 << 4)


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 64), (7, 96), (33, 128), (1025, 4128), (5, 4096)])
def test_quantize_ragged_shapes(rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    x = wl.f32_to_bf16_bits(rng.standard_t(3, size=(rows, cols)).astype(np.float32) * 0.5)
    for rule in RULES:
        gc, gs = _gpu_rows(x, rule)
        oc, os_ = oracle.quantize_rows(x, rule)
        np.testing.assert_array_equal(gs, os_)
        np.testing.assert_array_equal(gc, oc)


@pytest.mark.parametrize("log2n", [20, 24, 27, 30])
def test_quantize_sweep_student_t(log2n):
    """Quantize-sweep workload: 0.5 * StudentT(3), [2^k / 4096, 4096]; every byte
    compared up to 2^24 elements, 2048 seeded rows beyond that."""
    x = wl.student_t_matrix(1 << log2n, 4096, seed=0)
    xd = _dev(x)
    rng = np.random.default_rng(log2n)
    for rule in RULES:
        c, s = mx.mxattn_quantize(xd, rule)
        torch.cuda.synchronize()
        if log2n <= 24:
            rows = np.arange(x.shape[0])
        else:
            rows = np.sort(rng.choice(x.shape[0], 2048, replace=False))
            rows[-1] = x.shape[0] - 1
        idx = torch.from_numpy(rows).cuda()
        gc, gs = c[idx].cpu().numpy(), s[idx].cpu().numpy()
        oc, os_ = oracle.quantize_rows(x[rows], rule)
        np.testing.assert_array_equal(gs, os_)
        np.testing.assert_array_equal(gc, oc)
        del c, s
    del xd
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N", [1, 31, 32, 33, 100, 128, 129, 300, 4096])
@pytest.mark.parametrize("d", [64, 128])
def test_quantize_vt_matches_oracle(N, d):
    Q, K, V = wl.gaussian_qkv(1, 3, N, d, seed=N)
    V = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(V) * np.float32(3.0))
    for rule in RULES:
        gc, gs = mx.mxattn_quantize_vt(_dev(V), rule)
        torch.cuda.synchronize()
        oc, os_ = oracle.quantize_cols(V, rule)
        np.testing.assert_array_equal(gs.cpu().numpy(), os_)
        np.testing.assert_array_equal(gc.cpu().numpy(), oc)
