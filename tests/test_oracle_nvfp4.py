"""Pins of the oracle's NVFP4 comparison variant (CPU).

The MXAttention abstract compares against NVFP4 baselines without
defining them; the oracle's reading (oracle.c, "NVFP4 comparison variant") is
NVIDIA's NVFP4: E2M1 elements in blocks of 16, one E4M3 scale per block and a
per-(batch, head) fp32 scale g = 448 / amax, scale arithmetic in fp32.  The
pins below check it against a library routine (torch's float8_e4m3fn
conversion), closed forms, invariants and special cases.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import workloads as wl

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _torch_e4m3(v):
    return torch.tensor(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(0, 0x7F, dtype=np.uint8)
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(oracle.e4m3_decode(codes), ref)
    assert oracle.e4m3_decode([0x7E])[0] == 448.0 and oracle.e4m3_decode([1])[0] == 2.0 ** -9


def test_e4m3_encode_matches_torch_float8_rne():
    """Every E4M3 value, every midpoint (ties) and its fp32 neighbours, and random
    fp32 values below the overflow midpoint 464 round as torch's float8_e4m3fn cast."""
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    mids32 = mids.astype(np.float32)
    near = np.concatenate([np.nextafter(mids32, np.float32(0)), mids32, np.nextafter(mids32, np.float32(1e9))])
    rng = np.random.default_rng(0)
    rnd = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(463.0), 200_000)).astype(np.float32)
    v = np.concatenate([vals.astype(np.float32), near, rnd, np.float32([0.0, 2.0 ** -10, 463.99997])])
    np.testing.assert_array_equal(oracle.e4m3_encode(v.astype(np.float64)), _torch_e4m3(v))


def test_e4m3_encode_saturates_and_drops_sign():
    assert list(oracle.e4m3_encode([464.0, 470.0, 1e9, np.inf])) == [0x7E] * 4
    np.testing.assert_array_equal(oracle.e4m3_encode([-1.0, -0.0]), oracle.e4m3_encode([1.0, 0.0]))


def test_global_scale_is_fp32_448_over_amax():
    for amax in [1.0, 3.0, 0.1, 1e-3, 6e4, 2.0 ** -100, 0.0]:
        a = max(np.float32(amax), np.float32(2.0 ** -100))
        assert oracle.nvfp4_global(amax) == np.float32(448.0) / a


def _blocks(seed=0, n=4096):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 16)).astype(np.float32) * np.exp(rng.uniform(-8, 8, (n, 1))).astype(np.float32)
    x[:32] = 0.0
    x[32:64, 5] = 1e-30  # tiny blocks: their scale underflows to zero
    return wl.f32_to_bf16_bits(x)


def test_nvfp4_block_scale_is_the_e4m3_of_amax_times_g():
    x = _blocks()
    xf = wl.bf16_bits_to_f32(x)
    g = oracle.nvfp4_global(np.abs(xf).max())
    codes, scales = oracle.nvfp4_quantize_rows(x, g)
    prod = (np.abs(xf).max(axis=1) * np.float32(g)).astype(np.float32)
    np.testing.assert_array_equal(scales[:, 0], _torch_e4m3(np.minimum(prod, np.float32(448.0))))


def test_nvfp4_elements_are_nearest_grid_points_of_x_times_r():
    """Brute force over the 8 E2M1 magnitudes: each code is the nearest grid point of
    x * r (fp32, r = 6g / sb), ties to the even code; saturating at 6."""
    x = _blocks(1)
    xf = wl.bf16_bits_to_f32(x)
    g = oracle.nvfp4_global(np.abs(xf).max())
    codes, scales = oracle.nvfp4_quantize_rows(x, g)
    sbv = oracle.e4m3_decode(scales[:, 0]).astype(np.float32)
    live = sbv > 0
    r = (np.float32(6.0) * np.float32(g) / np.where(live, sbv, 1)).astype(np.float32)
    v = (xf * r[:, None]).astype(np.float32).astype(np.float64)
    c = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(x.shape)
    mag = c & 7
    d = np.abs(np.abs(v)[..., None] - E2M1)
    best = d.min(axis=-1)
    assert np.all((np.abs(np.abs(v) - E2M1[mag]) == best) | ~live[:, None] | (np.abs(v) >= 6))
    ties = (d == best[..., None]).sum(-1) == 2
    assert np.all((mag[ties & live[:, None]] % 2) == 0)
    assert np.all(mag[~live] == 0)
    np.testing.assert_array_equal(c >> 3, (xf < 0) | ((xf == 0) & np.signbit(xf)))


def test_nvfp4_block_maximum_lands_on_six():
    """With a normal E4M3 scale, sb is within 1/16 of amax * g, so the block maximum
    times r lies in [6 / (1 + 1/16), 6 / (1 - 1/16)] and always encodes as 6 (code 7)."""
    x = _blocks(2)
    xf = wl.bf16_bits_to_f32(x)
    g = oracle.nvfp4_global(np.abs(xf).max())
    codes, scales = oracle.nvfp4_quantize_rows(x, g)
    c = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(x.shape)
    normal = scales[:, 0] >= 0x08
    imax = np.abs(xf).argmax(axis=1)
    assert np.all((c[np.arange(len(x)), imax] & 7)[normal] == 7)


def test_nvfp4_equivariant_under_powers_of_two():
    x = _blocks(3, 512)
    xf = wl.bf16_bits_to_f32(x)
    base = oracle.nvfp4_quantize_rows(x, oracle.nvfp4_global(np.abs(xf).max()))
    for k in (-20, -3, 5, 17):
        y = wl.f32_to_bf16_bits(xf * np.float32(2.0 ** k))
        got = oracle.nvfp4_quantize_rows(y, oracle.nvfp4_global(np.abs(xf).max() * 2.0 ** k))
        np.testing.assert_array_equal(got[0], base[0])
        np.testing.assert_array_equal(got[1], base[1])


def test_nvfp4_ones_quantize_exactly():
    ones = wl.f32_to_bf16_bits(np.ones((4, 64), np.float32))
    g = oracle.nvfp4_global(1.0)
    codes, scales = oracle.nvfp4_quantize_rows(ones, g)
    assert np.all(codes == 0x77) and np.all(scales == 0x7E)
    np.testing.assert_array_equal(oracle.nvfp4_dequantize_rows(codes, scales, g), 1.0)


def test_nvfp4_cols_equal_rows_of_the_transpose():
    Q, _, V = wl.gaussian_qkv(1, 2, 70, 64, seed=4)
    g = oracle.nvfp4_head_globals(V)
    ct, st = oracle.nvfp4_quantize_cols(V, g)
    npad = 96
    for h in range(2):
        vt = np.zeros((64, npad), np.uint16)
        vt[:, :70] = V[0, h].T
        c, s = oracle.nvfp4_quantize_rows(vt, g[0, h])
        np.testing.assert_array_equal(ct[0, h], c)
        np.testing.assert_array_equal(st[0, h], s)


def _softmax_ref(q, k, v, scale):
    s = q @ k.T * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p / p.sum(axis=1, keepdims=True)) @ v


@pytest.mark.parametrize("kv_tile", [32, 64, 128])
def test_nvfp4_attention_without_quantization_is_softmax(kv_tile):
    Q, K, V = wl.gaussian_qkv(1, 1, 150, 64, seed=5)
    got = oracle.nvfp4_attention(Q, K, V, kv_tile, quant=False)[0, 0]
    f = lambda a: wl.bf16_bits_to_f32(a[0, 0]).astype(np.float64)  # noqa: E731
    np.testing.assert_allclose(got, _softmax_ref(f(Q), f(K), f(V), 1 / 8), rtol=0, atol=1e-12)


def test_nvfp4_attention_exact_p_is_softmax_of_dequantized_operands():
    Q, K, V = wl.gaussian_qkv(1, 1, 100, 64, seed=6)
    got = oracle.nvfp4_attention(Q, K, V, 64, p_quant=False)[0, 0]
    g = [oracle.nvfp4_head_globals(a)[0, 0] for a in (Q, K, V)]
    q = oracle.nvfp4_dequantize_rows(*oracle.nvfp4_quantize_rows(Q[0, 0], g[0]), g[0])
    k = oracle.nvfp4_dequantize_rows(*oracle.nvfp4_quantize_rows(K[0, 0], g[1]), g[1])
    ct, st = oracle.nvfp4_quantize_cols(V, np.float32(g[2]))
    vt = oracle.nvfp4_dequantize_rows(ct[0, 0], st[0, 0], g[2])[:, :100]
    np.testing.assert_allclose(got, _softmax_ref(q, k, vt.T, 1 / 8), rtol=0, atol=1e-12)


def test_nvfp4_attention_single_tile_p_blocks():
    """One key tile: O = sum q_j v_j / sum q_j with q the NVFP4 quantization of
    exp(s - max) per 16 keys (E4M3 scale via torch, E2M1 by brute force)."""
    Q, K, V = wl.gaussian_qkv(1, 1, 48, 64, seed=7)
    got = oracle.nvfp4_attention(Q, K, V, 64, p_quant=True)[0, 0]
    g = [oracle.nvfp4_head_globals(a)[0, 0] for a in (Q, K, V)]
    q = oracle.nvfp4_dequantize_rows(*oracle.nvfp4_quantize_rows(Q[0, 0], g[0]), g[0])
    k = oracle.nvfp4_dequantize_rows(*oracle.nvfp4_quantize_rows(K[0, 0], g[1]), g[1])
    ct, st = oracle.nvfp4_quantize_cols(V, np.float32(g[2]))
    v = oracle.nvfp4_dequantize_rows(ct[0, 0], st[0, 0], g[2])[:, :48].T
    s = q @ k.T / 8
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p = np.concatenate([p, np.zeros((48, 16))], axis=1)  # the tile's 64 columns, 48 valid
    qp = np.zeros_like(p)
    for b in range(4):
        blk = p[:, 16 * b:16 * b + 16]
        sbv = oracle.e4m3_decode(_torch_e4m3((blk.max(axis=1).astype(np.float32) * np.float32(448)).astype(np.float32)))
        r = np.where(sbv > 0, np.float32(2688) / np.where(sbv > 0, sbv, 1).astype(np.float32), 0).astype(np.float32)
        val = blk * r[:, None].astype(np.float64)
        d = np.abs(val[..., None] - E2M1)
        idx = d.argmin(-1)
        tie = (d == d.min(-1, keepdims=True)).sum(-1) == 2
        idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)
        idx = np.where(val >= 6, 7, idx)
        qp[:, 16 * b:16 * b + 16] = E2M1[idx] * sbv[:, None] / 2688.0
    qp = qp[:, :48]
    ref = (qp @ v) / qp.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_nvfp4_pnq_normalizes_by_construction():
    Q, K, _ = wl.gaussian_qkv(1, 1, 300, 64, seed=8)
    ones = wl.f32_to_bf16_bits(np.ones((1, 1, 300, 64), np.float32))
    on = oracle.nvfp4_attention(Q, K, ones, 128, pnq=True)
    off = oracle.nvfp4_attention(Q, K, ones, 128, pnq=False)
    np.testing.assert_allclose(on, 1.0, rtol=0, atol=1e-12)
    assert np.max(np.abs(off - 1.0)) > 1e-4


def test_nvfp4_special_cases():
    Q, _, V = wl.gaussian_qkv(1, 1, 64, 64, seed=9)
    zeros = np.zeros_like(Q)
    gv = oracle.nvfp4_head_globals(V)
    ct, st = oracle.nvfp4_quantize_cols(V, gv)
    vt = oracle.nvfp4_dequantize_rows(ct[0, 0], st[0, 0], gv[0, 0])[:, :64]
    o = oracle.nvfp4_attention(Q, zeros, V, 64)[0, 0]  # K = 0: equal scores, p = 1 -> 1 exactly
    np.testing.assert_allclose(o, np.broadcast_to(vt.mean(axis=1), o.shape), rtol=0, atol=1e-12)
    o1 = oracle.nvfp4_attention(Q[:, :, :1], Q[:, :, :1], V[:, :, :1], 64)[0, 0]
    g1 = oracle.nvfp4_head_globals(V[:, :, :1])
    c1, s1 = oracle.nvfp4_quantize_cols(V[:, :, :1], g1)  # N = 1: O = deq(V_0), V quantized along tokens
    v0 = oracle.nvfp4_dequantize_rows(c1[0, 0], s1[0, 0], g1[0, 0])[:, 0]
    np.testing.assert_allclose(o1, v0[None, :], rtol=0, atol=1e-12)
