"""Parity of the NVFP4 comparison variant (the NVFP4 baselines of the
MXAttention abstract, "MXAttention: Data-Free Optimal Scaling and
Pre-Normalization Quantization for MXFP4 Attention") with the CPU oracle.

Codes, E4M3 scales and second-level scales g are decided from bf16 inputs in
fp32 on both sides and must match bit for bit; O within the attention
tolerance (relative Frobenius <= 1e-3, max-abs <= 2e-2), P's codes being
decided in fp32 by the kernel and in fp64 by the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200 import workloads as wl

from test_attention_gpu import assert_close, sampled_rows
from test_quantize_gpu import _dev, _finite_patterns

pytestmark = pytest.mark.gpu


def _gpu_quantize(bits):
    c, s, gs = mx.mxattn_nvfp4_quantize(_dev(bits))
    torch.cuda.synchronize()
    return c.cpu().numpy(), s.cpu().numpy(), gs.cpu().numpy()


def _oracle_quantize(bits):
    amax = float(np.abs(wl.bf16_bits_to_f32(bits)).max()) if bits.size else 0.0
    g = oracle.nvfp4_global(amax)
    c, s = oracle.nvfp4_quantize_rows(bits, g)
    return c, s, np.float32(amax), g


def _check_standalone(bits):
    c, s, gs = _gpu_quantize(bits)
    oc, os_, amax, g = _oracle_quantize(bits)
    assert gs[0] == amax and gs[1] == g, (gs, amax, g)
    np.testing.assert_array_equal(s, os_)
    np.testing.assert_array_equal(c, oc)


def test_standalone_every_bf16_pattern_in_random_blocks():
    pats = _finite_patterns()
    rng = np.random.default_rng(0)
    x = rng.permutation(np.concatenate([pats, pats]))
    x = x[: len(x) // 64 * 64].reshape(-1, 64)
    _check_standalone(x)


@pytest.mark.parametrize("scale_exp", [-30, -8, 0, 9, 40])
def test_standalone_gaussian_blocks_over_magnitudes(scale_exp):
    rng = np.random.default_rng(scale_exp + 100)
    x = rng.standard_normal((1024, 256)).astype(np.float32)
    x *= np.exp(rng.uniform(-12, 12, (1024, 1))).astype(np.float32) * np.float32(2.0 ** scale_exp)
    _check_standalone(wl.f32_to_bf16_bits(x))


def test_standalone_student_t_and_edge_tensors():
    _check_standalone(wl.student_t_matrix(1 << 20, cols=4096, seed=3))
    _check_standalone(np.zeros((8, 32), dtype=np.uint16))                       # all zeros: g from the floor
    _check_standalone(wl.f32_to_bf16_bits(np.full((4, 16), -0.0, np.float32)))  # signed zeros
    tiny = np.zeros((4, 64), np.float32)
    tiny[:, 0] = 1000.0
    tiny[:, 16:32] = 1e-7                                                        # scales that round to 0
    _check_standalone(wl.f32_to_bf16_bits(tiny))


def _region(ws, name, B, H, N, d):
    off, size = mx.nvfp4_workspace_layout(B, H, N, d)[name]
    return ws[off: off + size].cpu().numpy()


def _unregroup_rows(sf, BH, N, d):
    """Regrouped NVFP4 Q/K scales [BH, G, (d/64)*512] -> row-major [BH, N, d/16]."""
    G = (N + 127) // 128
    chunks = sf.reshape(BH, G, d // 64 * 512)
    r = np.arange(N)
    m = r % 128
    out = np.empty((BH, N, d // 16), dtype=np.uint8)
    for j in range(d // 16):
        out[:, :, j] = chunks[:, r // 128, (j // 4) * 512 + (m % 32) * 16 + (m // 32) * 4 + j % 4]
    return out


def _unregroup_vt(sf, BH, N, d):
    """Regrouped NVFP4 V^T scales [BH, G, 1024] -> row-major [BH, d, Npad/16]."""
    G = (N + 127) // 128
    nb = (N + 31) // 32 * 2
    chunks = sf.reshape(BH, G, 1024)
    tb = np.arange(nb)
    out = np.empty((BH, d, nb), dtype=np.uint8)
    for c in range(d):
        out[:, c, :] = chunks[:, tb // 8, ((tb % 8) // 4) * 512 + (c % 32) * 16 + (c // 32) * 4 + tb % 4]
    return out


def check_workspace(ws, Q, K, V):
    """NVFP4 workspace codes, scales and g of Q, K, V^T == oracle, bit for bit."""
    B, H, N, d = Q.shape
    BH = B * H
    npad = (N + 31) // 32 * 32
    gq, gk, gv = (oracle.nvfp4_head_globals(x).ravel() for x in (Q, K, V))
    g = _region(ws, "g", B, H, N, d).view(np.float32).reshape(3, BH)
    np.testing.assert_array_equal(g[0], gq)
    np.testing.assert_array_equal(g[1], gk)
    np.testing.assert_array_equal(g[2], gv)
    qc = _region(ws, "q_codes", B, H, N, d).reshape(BH, N, d // 2)
    kc = _region(ws, "k_codes", B, H, N, d).reshape(BH, N, d // 2)
    vc = _region(ws, "vt_codes", B, H, N, d).reshape(BH, d, npad // 2)
    qs = _unregroup_rows(_region(ws, "q_sf", B, H, N, d), BH, N, d)
    ks = _unregroup_rows(_region(ws, "k_sf", B, H, N, d), BH, N, d)
    vs = _unregroup_vt(_region(ws, "vt_sf", B, H, N, d), BH, N, d)
    Qf, Kf, Vf = (x.reshape(BH, N, d) for x in (Q, K, V))
    for bh in range(BH):
        oc, os_ = oracle.nvfp4_quantize_rows(Qf[bh], gq[bh])
        np.testing.assert_array_equal(qc[bh], oc)
        np.testing.assert_array_equal(qs[bh], os_)
        oc, os_ = oracle.nvfp4_quantize_rows(Kf[bh], gk[bh])
        np.testing.assert_array_equal(kc[bh], oc)
        np.testing.assert_array_equal(ks[bh], os_)
        oc, os_ = oracle.nvfp4_quantize_cols(Vf[bh], gv[bh])
        np.testing.assert_array_equal(vc[bh], oc)
        np.testing.assert_array_equal(vs[bh], os_)


def run_nv(Q, K, V, T, pnq=True, scale=0.0):
    B, H, N, d = Q.shape
    ws = mx.new_nvfp4_workspace(B, H, N, d)
    O = mx.mxattn_nvfp4_forward(_dev(Q), _dev(K), _dev(V), T, pnq, scale, workspace=ws)
    assert mx.mxattn_workspace_status(ws) == 0
    return O.cpu().numpy().astype(np.float64), ws


@pytest.mark.parametrize("pnq", [True, False])
def test_tiny_config(pnq):
    w = wl.WORKLOADS["tiny"]
    Q, K, V = wl.make_qkv(w, seed=0)
    O, ws = run_nv(Q, K, V, w.kv_tile, pnq)
    assert_close(O, oracle.nvfp4_attention(Q, K, V, w.kv_tile, pnq=pnq), f"nvfp4 tiny pnq={pnq}")
    check_workspace(ws, Q, K, V)


@pytest.mark.parametrize("N", [1, 33, 129, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [64, 128])
def test_ragged_shapes(N, d, T):
    Q, K, V = wl.gaussian_qkv(1, 3, N, d, seed=N + d + T)
    V = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(V) * np.float32(3.0))
    for pnq in (True, False):
        O, ws = run_nv(Q, K, V, T, pnq)
        assert_close(O, oracle.nvfp4_attention(Q, K, V, T, pnq=pnq), f"nvfp4 N={N} d={d} T={T} pnq={pnq}")
    check_workspace(ws, Q, K, V)


def test_pnq_ones_and_zero_keys():
    Q, K, _ = wl.gaussian_qkv(1, 2, 500, 128, seed=5)
    ones = wl.f32_to_bf16_bits(np.ones((1, 2, 500, 128), np.float32))
    O, _ = run_nv(Q, K, ones, 128, True)
    np.testing.assert_allclose(O, 1.0, rtol=0, atol=2e-6)  # PNQ: the row sum is the tensor core's own sum
    _, _, V = wl.gaussian_qkv(1, 2, 500, 128, seed=6)
    O, _ = run_nv(Q, np.zeros_like(K), V, 128, True)
    assert_close(O, oracle.nvfp4_attention(Q, np.zeros_like(K), V, 128, pnq=True), "nvfp4 K=0")


def test_prepare_attend_equals_forward():
    Q, K, V = wl.gaussian_qkv(1, 2, 700, 128, seed=7)
    O, _ = run_nv(Q, K, V, 128, True)
    ws = mx.mxattn_nvfp4_prepare(_dev(Q), _dev(K), _dev(V))
    O2 = mx.mxattn_nvfp4_attend(ws, 1, 2, 700, 128, 128, True).cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(O, O2)


def test_outlier_and_video_recipes_sampled_rows():
    Q, K, V = wl.outlier_qkv(1, 2, 4096, 128, seed=0)
    O, ws = run_nv(Q, K, V, 128, True)
    rows = sampled_rows(4096, 96, 1)
    assert_close(O[:, :, rows], oracle.nvfp4_attention(Q, K, V, 128, pnq=True, rows=rows), "nvfp4 outlier")
    check_workspace(ws, Q, K, V)
    vid = wl.WORKLOADS["video_dit"]
    Q, K, V = wl.video_dit_qkv(1, 2, vid.frames, vid.rows, vid.cols, vid.d, seed=3)
    O, ws = run_nv(Q, K, V, 128, True)
    rows = sampled_rows(vid.N, 24, 2)
    assert_close(O[:, :, rows], oracle.nvfp4_attention(Q, K, V, 128, pnq=True, rows=rows), "nvfp4 video-DiT")
    check_workspace(ws, Q, K, V)
