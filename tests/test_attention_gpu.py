"""Parity of the fused MXFP4 attention (UOS + PNQ) with the CPU oracle.

Method: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
Quantization for MXFP4 Attention", abstract.  Tolerance for O (fp32 kernel vs
fp64 oracle, same kv_tile and ascending tile order): relative Frobenius error
<= 1e-3 and max absolute error <= 2e-2.  Q/K/V^T codes and scales (in the
workspace) must match the oracle bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_FROB = 1e-3
MAX_ABS = 2e-2


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def run_forward(Q, K, V, T, pnq=True, rule="uos", scale=0.0):
    B, H, N, d = Q.shape
    ws = mx.new_workspace(B, H, N, d)
    O = mx.mxattn_forward(_dev(Q), _dev(K), _dev(V), T, pnq, rule, scale, workspace=ws)
    assert mx.mxattn_workspace_status(ws) == 0
    return O.cpu().numpy().astype(np.float64), ws


def assert_close(O, R, what=""):
    assert np.all(np.isfinite(O)), what
    rel = np.linalg.norm(O - R) / np.linalg.norm(R)
    mabs = float(np.max(np.abs(O - R)))
    assert rel <= REL_FROB and mabs <= MAX_ABS, f"{what}: rel-Frobenius {rel:.3e}, max-abs {mabs:.3e}"
    print(f"[parity] {what}: rel-Frobenius {rel:.3e}, max-abs {mabs:.3e}")
    return rel, mabs


def _region(ws, name, B, H, N, d):
    off, size = mx.workspace_layout(B, H, N, d)[name]
    return ws[off: off + size].cpu().numpy()


def _unregroup_rows(sf, BH, N, kb):
    """Regrouped scales [BH, G, 512] -> row-major [BH, N, kb]."""
    G = (N + 127) // 128
    chunks = sf.reshape(BH, G, 512)
    r = np.arange(N)
    m = r % 128
    out = np.empty((BH, N, kb), dtype=np.uint8)
    for k in range(kb):
        out[:, :, k] = chunks[:, r // 128, (m % 32) * 16 + (m // 32) * 4 + k]
    return out


def _unregroup_vt(sf, BH, N, d):
    """Regrouped V^T scales [BH, G, 512] -> row-major [BH, d, Npad/32]."""
    G = (N + 127) // 128
    nb = (N + 31) // 32
    chunks = sf.reshape(BH, G, 512)
    tb = np.arange(nb)
    out = np.empty((BH, d, nb), dtype=np.uint8)
    for c in range(d):
        out[:, c, :] = chunks[:, tb // 4, (c % 32) * 16 + (c // 32) * 4 + tb % 4]
    return out


def check_codes(ws, Q, K, V, rule, heads=None):
    """Workspace Q/K/V^T codes and scales == oracle, bit for bit (optionally on a subset of heads)."""
    B, H, N, d = Q.shape
    BH = B * H
    hs = np.arange(BH) if heads is None else np.asarray(heads)
    qc = _region(ws, "q_codes", B, H, N, d).reshape(BH, N, d // 2)
    kc = _region(ws, "k_codes", B, H, N, d).reshape(BH, N, d // 2)
    npad = (N + 31) // 32 * 32
    vc = _region(ws, "vt_codes", B, H, N, d).reshape(BH, d, npad // 2)
    qs = _unregroup_rows(_region(ws, "q_sf", B, H, N, d), BH, N, d // 32)
    ks = _unregroup_rows(_region(ws, "k_sf", B, H, N, d), BH, N, d // 32)
    vs = _unregroup_vt(_region(ws, "vt_sf", B, H, N, d), BH, N, d)
    Qf, Kf, Vf = (x.reshape(BH, N, d) for x in (Q, K, V))
    for bh in hs:
        oc, os_ = oracle.quantize_rows(Qf[bh], rule)
        np.testing.assert_array_equal(qc[bh], oc)
        np.testing.assert_array_equal(qs[bh], os_)
        oc, os_ = oracle.quantize_rows(Kf[bh], rule)
        np.testing.assert_array_equal(kc[bh], oc)
        np.testing.assert_array_equal(ks[bh], os_)
        oc, os_ = oracle.quantize_cols(Vf[bh], rule)
        np.testing.assert_array_equal(vc[bh], oc)
        np.testing.assert_array_equal(vs[bh], os_)


def sampled_rows(N, n, seed):
    """n seeded random query rows plus the first and last rows and the edges of the first and last tiles."""
    rng = np.random.default_rng(seed)
    edges = {0, N - 1, min(127, N - 1), min(128, N - 1), (N - 1) // 128 * 128}
    return np.array(sorted(edges | set(rng.choice(N, min(n, N), replace=False).tolist())), dtype=np.int64)


# ---------------------------------------------------------------------------- small configurations


@pytest.mark.parametrize("rule", ["ocp", "uos"])
@pytest.mark.parametrize("pnq", [True, False])
def test_tiny_config_all_variants(rule, pnq):
    w = wl.WORKLOADS["tiny"]
    Q, K, V = wl.make_qkv(w, seed=0)
    O, ws = run_forward(Q, K, V, w.kv_tile, pnq, rule)
    R = oracle.attention(Q, K, V, w.kv_tile, rule=rule, pnq=pnq)
    assert_close(O, R, f"tiny {rule} pnq={pnq}")
    check_codes(ws, Q, K, V, rule)


@pytest.mark.parametrize("N", [1, 33, 100, 129, 255, 257, 640])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [64, 128])
def test_ragged_shapes(N, d, T):
    Q, K, V = wl.gaussian_qkv(2, 3, N, d, seed=N + d + T)
    Q = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(Q) * np.float32(2.0))
    for rule, pnq in (("uos", True), ("ocp", False)):
        O, ws = run_forward(Q, K, V, T, pnq, rule)
        R = oracle.attention(Q, K, V, T, rule=rule, pnq=pnq)
        assert_close(O, R, f"N={N} d={d} T={T} {rule} pnq={pnq}")
    check_codes(ws, Q, K, V, "ocp")


def test_more_heads_than_a_grid_dimension():
    """B*H above 65,535 (one fused preparation launch, one attention CTA per head and
    tile pair): sampled heads, including both sides of 65,536, against the oracle."""
    B, H, N, d, T = 1, 66000, 3, 64, 64
    Q, K, V = wl.gaussian_qkv(B, H, N, d, seed=66)
    O, ws = run_forward(Q, K, V, T, True, "uos")
    heads = [0, 1, 4097, 65534, 65535, 65536, 65537, H - 1]
    check_codes(ws, Q, K, V, "uos", heads=heads)
    sel = lambda X: X[:, heads]
    R = oracle.attention(sel(Q), sel(K), sel(V), T, rule="uos", pnq=True)
    assert_close(O[:, heads], R, "B*H = 66000, sampled heads")


def test_explicit_softmax_scale():
    Q, K, V = wl.gaussian_qkv(1, 2, 300, 64, seed=11)
    O, _ = run_forward(Q, K, V, 64, True, "uos", scale=0.3)
    R = oracle.attention(Q, K, V, 64, rule="uos", pnq=True, scale=0.3)
    assert_close(O, R, "scale=0.3")


def test_forward_quantized_matches_forward_bitwise():
    Q, K, V = wl.gaussian_qkv(1, 4, 700, 128, seed=12)
    O1, _ = run_forward(Q, K, V, 128, True, "uos")
    q, k, v = _dev(Q), _dev(K), _dev(V)
    qc, qs = mx.mxattn_quantize(q, "uos")
    kc, ks = mx.mxattn_quantize(k, "uos")
    vc, vs = mx.mxattn_quantize_vt(v, "uos")
    ws = mx.new_workspace(1, 4, 700, 128)
    O2 = mx.mxattn_forward_quantized(qc, qs, kc, ks, vc, vs, 1, 4, 700, 128, 128, True, "uos", workspace=ws)
    assert mx.mxattn_workspace_status(ws) == 0
    np.testing.assert_array_equal(O2.cpu().numpy(), O1.astype(np.float32))


@pytest.mark.parametrize("N,d,T,rule", [(700, 128, 128, "uos"), (129, 64, 64, "ocp"), (300, 64, 128, 6.5),
                                          (1, 128, 64, "uos"), (1000, 128, 128, "ocp")])
def test_forward_matches_prepare_attend_and_fills_the_workspace(N, d, T, rule):
    """mxattn_forward and mxattn_prepare + mxattn_attend give the same O and the
    same workspace (Q/K/V^T codes and scales) bit for bit, starting from two
    different fill bytes, so every byte of those regions is written."""
    Q, K, V = wl.gaussian_qkv(2, 3, N, d, seed=13)
    q, k, v = _dev(Q), _dev(K), _dev(V)
    ws1 = mx.new_workspace(2, 3, N, d)
    ws2 = mx.new_workspace(2, 3, N, d)
    ws1.fill_(0x5A)  # different fills: a byte either path leaves unwritten shows up as a difference
    ws2.fill_(0xA5)
    O1 = mx.mxattn_forward(q, k, v, T, True, rule, 0.0, workspace=ws1)
    mx.mxattn_prepare(q, k, v, rule, ws2)
    O2 = torch.empty_like(O1)
    mx.mxattn_attend(ws2, 2, 3, N, d, T, True, rule, 0.0, O2)
    torch.cuda.synchronize()
    assert mx.mxattn_workspace_status(ws1) == 0 and mx.mxattn_workspace_status(ws2) == 0
    assert torch.equal(O1, O2)
    for name in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"):
        a, b = _region(ws1, name, 2, 3, N, d), _region(ws2, name, 2, 3, N, d)
        np.testing.assert_array_equal(a, b, err_msg=name)


@pytest.mark.parametrize("d,T", [(64, 64), (128, 128), (128, 64)])
def test_forward_quantized_on_oracle_operands(d, T):
    """The attention step alone, fed operands quantized by the oracle."""
    N, H = 517, 2
    Q, K, V = wl.gaussian_qkv(1, H, N, d, seed=13)
    qc, qs = oracle.quantize_rows(Q, "uos")
    kc, ks = oracle.quantize_rows(K, "uos")
    vc, vs = oracle.quantize_cols(V, "uos")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    ws = mx.new_workspace(1, H, N, d)
    O = mx.mxattn_forward_quantized(t(qc), t(qs), t(kc), t(ks), t(vc), t(vs), 1, H, N, d, T, True, "uos",
                                    workspace=ws)
    assert mx.mxattn_workspace_status(ws) == 0
    R = oracle.attention(Q, K, V, T, rule="uos", pnq=True)
    assert_close(O.cpu().numpy().astype(np.float64), R, "forward_quantized")


def test_pnq_normalization_on_gpu():
    """V = 1: with PNQ the tensor-core row sum and O accumulate the same quantized
    exponentials, so O == 1; without PNQ it is not."""
    N, d = 1000, 128
    Q, K, _ = wl.gaussian_qkv(1, 2, N, d, seed=14)
    Q = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(Q) * np.float32(3.0))
    ones = np.full_like(Q, 0x3F80)
    O, _ = run_forward(Q, K, ones, 128, True, "uos")
    np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-6)
    O2, _ = run_forward(Q, K, ones, 128, False, "uos")
    assert np.max(np.abs(O2 - 1.0)) > 1e-3
    R2 = oracle.attention(Q, K, ones, 128, rule="uos", pnq=False)
    assert_close(O2, R2, "ones pnq off")


def test_zero_keys_give_column_mean():
    N, d = 333, 64
    Q, _, V = wl.gaussian_qkv(1, 1, N, d, seed=15)
    K = np.zeros_like(Q)
    O, _ = run_forward(Q, K, V, 64, True, "uos")
    vc, vs = oracle.quantize_cols(V, "uos")
    mean = oracle.dequantize_rows(vc, vs)[0, 0][:, :N].mean(axis=1)
    np.testing.assert_allclose(O[0, 0], np.broadcast_to(mean, (N, d)), rtol=1e-5, atol=1e-6)


def test_deterministic():
    Q, K, V = wl.gaussian_qkv(1, 2, 1500, 128, seed=16)
    O1, _ = run_forward(Q, K, V, 128, True, "uos")
    O2, _ = run_forward(Q, K, V, 128, True, "uos")
    np.testing.assert_array_equal(O1, O2)


# ---------------------------------------------------------------------------- workload configurations


def test_outlier_config():
    w = wl.WORKLOADS["outlier"]
    Q, K, V = wl.make_qkv(w, seed=0)
    for rule, pnq in (("uos", True), ("ocp", False)):
        O, ws = run_forward(Q, K, V, w.kv_tile, pnq, rule)
        check_codes(ws, Q, K, V, rule)
        rows = [np.arange(w.N)] + [sampled_rows(w.N, 256, h) for h in range(1, w.H)]
        for h in range(w.H):
            R = oracle.attention(Q[:, h:h + 1], K[:, h:h + 1], V[:, h:h + 1], w.kv_tile, rule=rule, pnq=pnq,
                                 rows=rows[h])
            assert_close(O[:, h:h + 1, rows[h]], R, f"outlier head {h} {rule} pnq={pnq}")


@pytest.mark.parametrize("name,head0_all_rows,rows_per_head", [("video_dit", True, 256),
                                                                 ("long_video_dit", False, 64)])
def test_video_dit_configs_full_size(name, head0_all_rows, rows_per_head):
    """Full-size workloads in the launch configuration the benchmark times:
    every Q/K/V^T code and scale bit-exact; O on every row of head 0 (video-DiT)
    and on seeded sampled rows (plus the tile edges) of every other head."""
    w = wl.WORKLOADS[name]
    Q, K, V = wl.make_qkv(w, seed=0)
    O, ws = run_forward(Q, K, V, w.kv_tile, True, "uos")
    check_codes(ws, Q, K, V, "uos")
    worst = 0.0
    for h in range(w.H):
        rows = np.arange(w.N) if (h == 0 and head0_all_rows) else sampled_rows(w.N, rows_per_head, 100 + h)
        R = oracle.attention(Q[:, h:h + 1], K[:, h:h + 1], V[:, h:h + 1], w.kv_tile, rule="uos", pnq=True,
                             rows=rows)
        rel, _ = assert_close(O[:, h:h + 1, rows], R, f"{name} head {h} ({len(rows)} rows)")
        worst = max(worst, rel)
    print(f"[parity] {name}: worst per-head rel-Frobenius {worst:.3e}")
    del ws
    torch.cuda.empty_cache()


def test_status_string_roundtrip():
    assert mx.mxattn_status_string(0) == "ok"
    assert "timed out" in mx.mxattn_status_string(4)
    assert math.isfinite(mx.mxattn_workspace_size(1, 40, 32760, 128))


@pytest.mark.parametrize("chunks,groups", [(1, None), (3, None), (8, None), (100, None), (16, [4, 1, 5]), (16, [10])])
def test_attention_from_host_pipeline_matches_forward(chunks, groups):
    """The host-to-host call (head groups pipelined over three streams, the
    default ramped schedule or explicit group sizes) gives the same O as one
    mxattn_forward on device tensors, bit for bit."""
    Q, K, V = wl.gaussian_qkv(2, 5, 300, 128, seed=31)
    ref, _ = run_forward(Q, K, V, 128, True, "uos")
    host = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()  # noqa: E731
    out = mx.attention_from_host(host(Q), host(K), host(V), 128, True, "uos", chunks=chunks, groups=groups)
    torch.cuda.current_stream().synchronize()
    np.testing.assert_array_equal(out.numpy().astype(np.float64), ref)


def test_forward_host_c_abi_matches_forward():
    """mxattn_forward_host called through the C ABI on pinned host buffers (both
    rules, PNQ on and off, d = 64 and 128, default and explicit group schedules)
    writes the same O as mxattn_forward on device tensors, bit for bit."""
    import ctypes

    for (B, H, N, d, T, pnq, rule, groups) in ((1, 6, 1000, 128, 128, True, "uos", None),
                                               (2, 3, 333, 64, 64, False, "ocp", [2, 1, 3]),
                                               (1, 1, 77, 128, 64, True, "ocp", None)):
        Q, K, V = wl.gaussian_qkv(B, H, N, d, seed=41 + N)
        ref, _ = run_forward(Q, K, V, T, pnq, rule)
        host = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()  # noqa: E731
        qh, kh, vh = host(Q), host(K), host(V)
        oh = torch.full((B, H, N, d), float("nan"), dtype=torch.float32).pin_memory()
        dev = [torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
        od = torch.empty((B, H, N, d), dtype=torch.float32, device="cuda")
        arr = None if groups is None else (ctypes.c_int * len(groups))(*groups)
        ng = 0 if groups is None else len(groups)
        wsb = mx.lib().mxattn_forward_host_workspace_size(B, H, N, d, arr, ng)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        st = mx.lib().mxattn_forward_host(p(qh), p(kh), p(vh), B, H, N, d, T, int(pnq), mx.RULES[rule],
                                          ctypes.c_float(0.0), p(oh), p(dev[0]), p(dev[1]), p(dev[2]), p(od), p(ws),
                                          wsb, arr, ng, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, mx.status_string(st)
        torch.cuda.current_stream().synchronize()
        assert mx.mxattn_workspace_status(ws) == 0
        np.testing.assert_array_equal(oh.numpy().astype(np.float64), ref)


def test_attention_from_host_rejects_bad_groups():
    Q, K, V = wl.gaussian_qkv(1, 3, 64, 64, seed=32)
    host = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()  # noqa: E731
    for groups in ([1, 1], [2, 2], [3, 0]):
        with pytest.raises(ValueError):
            mx.attention_from_host(host(Q), host(K), host(V), 64, True, "uos", groups=groups)
