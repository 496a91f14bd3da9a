"""Pins for the CPU oracle, checked against what the MXAttention abstract and
the mathematics fix (no GPU).

Source: "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
Quantization for MXFP4 Attention", abstract: MXFP4 (OCP MX) operands, the UOS
boundary Qmax = 7.25, and PNQ (the exponentials exp(s - m) are quantized before
the row sum, so the sum is built from the same values that weight V and the
normalization holds by construction).

Each check is independent of the oracle's own code: brute-force argmin for the
rounding, closed forms on the bit patterns for the scale rules, numpy's direct
softmax for the loop, hand-derived values for small cases.
"""
import math
import os

import numpy as np
import pytest

import oracle
from mxfp4_microscaled_quantization_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _bits(vals):
    return wl.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


# ----------------------------------------------------------------------------- E2M1 element format


def test_e2m1_decode_matches_grid_table():
    for code_s, val_s in _read_golden("e2m1_grid.txt"):
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e2m1_decode([code])[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e2m1_round_trip_all_codes():
    vals = oracle.e2m1_decode(np.arange(16))
    assert list(oracle.e2m1_encode(vals)) == list(range(16))


def test_e2m1_rounding_golden_cases():
    for v_s, code_s in _read_golden("e2m1_rounding.txt"):
        assert oracle.e2m1_encode([float(v_s)])[0] == int(code_s, 16), v_s


def _brute_force_e2m1(v):
    """Nearest grid magnitude by exhaustive distance over the 8 magnitudes,
    ties to the even code, saturating at 6; the sign bit always kept."""
    a = np.abs(v)
    dist = np.abs(a[:, None] - GRID[None, :])
    best = dist.min(axis=1, keepdims=True)
    is_best = dist == best
    n_best = is_best.sum(axis=1)
    idx = np.argmax(is_best, axis=1)  # first (smaller) candidate
    tie = n_best > 1
    # on a tie the candidates are idx and idx+1: keep the even one
    idx = np.where(tie & (idx % 2 == 1), idx + 1, idx)
    idx = np.where(a >= 6.0, 7, idx)
    return (np.signbit(v).astype(np.uint8) << 3) | idx.astype(np.uint8)


def test_e2m1_rounding_brute_force_all_bf16_patterns():
    bits = np.arange(1 << 16, dtype=np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite patterns only
    v = wl.bf16_bits_to_f32(bits).astype(np.float64)
    for shift in (-130, -3, -1, 0, 1, 2, 3, 5):
        x = np.ldexp(v, shift)
        x = x[np.isfinite(x)]
        np.testing.assert_array_equal(oracle.e2m1_encode(x), _brute_force_e2m1(x))


def test_e2m1_error_bound_unclipped():
    """|x - deq| <= half the local grid step for |x| <= 6 (nearest rounding)."""
    rng = np.random.default_rng(1)
    x = rng.uniform(-6, 6, 100000)
    d = oracle.e2m1_decode(oracle.e2m1_encode(x))
    step = np.where(np.abs(x) < 2, 0.5, np.where(np.abs(x) < 4, 1.0, 2.0))
    assert np.all(np.abs(x - d) <= step / 2 + 1e-15)


# ----------------------------------------------------------------------------- scale rules (OCP, UOS)


def test_scale_rules_golden_cases():
    for h, _val, e_ocp, e_uos in _read_golden("scale_rules.txt"):
        a = float(wl.bf16_bits_to_f32(np.array([int(h, 16)], dtype=np.uint16))[0])
        assert oracle.scale_exponent([a], "ocp")[0] == int(e_ocp), h
        assert oracle.scale_exponent([a], "uos")[0] == int(e_uos), h


def _all_positive_finite_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint16)  # 0x0001 .. 0x7F7F
    return bits, wl.bf16_bits_to_f32(bits).astype(np.float64)


def test_ocp_rule_invariant_all_bf16():
    """OCP: amax / 2^e in [4, 8) for every positive finite bf16 amax not clamped at -127."""
    bits, a = _all_positive_finite_bf16()
    e = oracle.scale_exponent(a, "ocp").astype(np.int64)
    r = np.ldexp(a, -e)
    free = e > -127
    assert np.all((r[free] >= 4) & (r[free] < 8))
    assert np.all(r[~free] < 8)  # clamped blocks never exceed the top binade


def test_uos_rule_invariant_and_minimality_all_bf16():
    """UOS: amax / 2^e <= 7.25 (abstract's Qmax) and amax / 2^(e-1) > 7.25 (smallest such e)."""
    bits, a = _all_positive_finite_bf16()
    e = oracle.scale_exponent(a, "uos").astype(np.int64)
    assert np.all(np.ldexp(a, -e) <= 7.25)
    free = e > -127
    assert np.all(np.ldexp(a[free], -(e[free] - 1)) > 7.25)


def test_uos_minus_ocp_closed_form_on_bits():
    """e_UOS - e_OCP = [mu > 1.8125] with amax = mu * 2^k, mu in [1, 2):
    on bf16 bits, mantissa field > 0x68 (7.25 / 4 = 1.8125 = 1 + 0x68/128)."""
    bits, a = _all_positive_finite_bf16()
    normal = (bits >> 7) > 1  # exponent field >= 2 keeps both rules off the clamp
    e_o = oracle.scale_exponent(a, "ocp").astype(np.int64)
    e_u = oracle.scale_exponent(a, "uos").astype(np.int64)
    expect = ((bits & 0x7F) > 0x68).astype(np.int64)
    np.testing.assert_array_equal((e_u - e_o)[normal], expect[normal])
    exp_field = (bits >> 7).astype(np.int64)
    np.testing.assert_array_equal(e_o[normal], (exp_field - 127 - 2)[normal])


def test_uos_clip_error_bound():
    """Under UOS the clipped part of a block's maximum is at most (7.25 - 6) * 2^e."""
    bits, a = _all_positive_finite_bf16()
    e = oracle.scale_exponent(a, "uos").astype(np.int64)
    deq = np.ldexp(oracle.e2m1_decode(oracle.e2m1_encode(np.ldexp(a, -e))), e)
    assert np.all(a - deq <= np.ldexp(1.25, e) * (1 + 1e-12))


# ----------------------------------------------------------------------------- scale boundary Qmax (sweep of the UOS family)

QMAX_SWEEP = [4.5, 5.0, 6.0, 6.5, 7.0, 7.25, 7.5, 7.75, 7.875]


def test_qmax_rule_golden_cases():
    for q, h, _val, e in _read_golden("qmax_rules.txt"):
        a = float(wl.bf16_bits_to_f32(np.array([int(h, 16)], dtype=np.uint16))[0])
        assert oracle.scale_exponent([a], float(q))[0] == int(e), (q, h)


@pytest.mark.parametrize("q", QMAX_SWEEP)
def test_qmax_rule_invariant_and_minimality_all_bf16(q):
    """Boundary rule: amax / 2^e <= Qmax and amax / 2^(e-1) > Qmax for every
    positive finite bf16 amax whose exponent is not clamped."""
    bits, a = _all_positive_finite_bf16()
    e = oracle.scale_exponent(a, q).astype(np.int64)
    assert np.all(np.ldexp(a, -e) <= q)
    free = e > -127
    assert np.all(np.ldexp(a[free], -(e[free] - 1)) > q)


@pytest.mark.parametrize("q", QMAX_SWEEP)
def test_qmax_minus_ocp_closed_form_on_bits(q):
    """With amax = mu * 2^k (mu in [1, 2)) and Qmax in (4, 8), the boundary rule
    gives k - 2 + [mu > Qmax/4]: on bf16 bits, mantissa field > floor((Qmax/4 - 1) * 128)."""
    bits, a = _all_positive_finite_bf16()
    normal = (bits >> 7) > 1
    e_o = oracle.scale_exponent(a, "ocp").astype(np.int64)
    e_q = oracle.scale_exponent(a, q).astype(np.int64)
    thresh = int(np.floor((q / 4 - 1) * 128))
    expect = ((bits & 0x7F) > thresh).astype(np.int64)
    np.testing.assert_array_equal((e_q - e_o)[normal], expect[normal])


def test_qmax_rule_contains_uos_and_tends_to_ocp():
    """Qmax = 7.25 is the UOS rule; a boundary just below 8 gives the OCP exponent
    for every bf16 maximum (mu < 2 <= Qmax/4 never holds, and mu * 2^k <=
    Qmax * 2^(k-3) would need mu < 1), and Qmax = 8 names OCP itself."""
    bits, a = _all_positive_finite_bf16()
    np.testing.assert_array_equal(oracle.scale_exponent(a, 7.25), oracle.scale_exponent(a, "uos"))
    np.testing.assert_array_equal(oracle.scale_exponent(a, 8.0), oracle.scale_exponent(a, "ocp"))
    near = oracle.scale_exponent(a, 8.0 - 2.0 ** -20)
    np.testing.assert_array_equal(near, oracle.scale_exponent(a, "ocp"))


def test_qmax_at_six_never_saturates():
    """Qmax = 6 (the largest E2M1 magnitude): every scaled element is <= 6, so no
    element clips and the error of each element is at most half a grid step."""
    bits, a = _all_positive_finite_bf16()
    e = oracle.scale_exponent(a, 6.0).astype(np.int64)
    r = np.ldexp(a, -e)
    assert np.all(r <= 6.0)
    deq = np.ldexp(oracle.e2m1_decode(oracle.e2m1_encode(r)), e)
    free = e > -127
    # grid spacing at r: 0.5 below 2, 1 in [2, 4), 2 in [4, 6]
    step = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    assert np.all(np.abs(a - deq)[free] <= np.ldexp(step / 2, e)[free] * (1 + 1e-12))


@pytest.mark.parametrize("q", [6.0, 7.5])
def test_qmax_attention_keeps_pnq_normalization(q):
    """PNQ's row sum is built from the quantized weights whatever the boundary:
    V = 1 gives O = 1 exactly (to rounding)."""
    N, d = 200, 64
    Q, K, _ = wl.gaussian_qkv(1, 1, N, d, seed=16)
    Q = _bits(wl.bf16_bits_to_f32(Q) * 3)
    ones = np.full((1, 1, N, d), 0x3F80, dtype=np.uint16)
    np.testing.assert_allclose(oracle.attention(Q, K, ones, 64, rule=q, pnq=True), 1.0, rtol=0, atol=1e-12)


def test_qmax_rule_rejects_boundaries_outside_the_family():
    for q in (4.0, 3.0, 8.5, 16.0):
        with pytest.raises(ValueError):
            oracle.scale_exponent([1.0], q)


# ----------------------------------------------------------------------------- block quantization


def test_quantize_rows_layout_hand_case():
    row = np.zeros(32, dtype=np.float32)
    row[0], row[1], row[2], row[3] = 6.0, -0.5, 1.0, -6.0
    codes, scales = oracle.quantize_rows(_bits(row)[None, :], "uos")
    # amax 6 -> e = 0 under both rules (6 <= 7.25; floor(log2 6) - 2 = 0)
    assert scales[0, 0] == 127
    assert codes[0, 0] == (0x7 | (0x9 << 4))  # element 0 low nibble, element 1 high nibble
    assert codes[0, 1] == (0x2 | (0xF << 4))
    assert np.all(codes[0, 2:] == 0)


@pytest.mark.parametrize("rule", ["ocp", "uos"])
def test_quantize_equivariance_power_of_two(rule):
    """The abstract presents UOS as needing no calibration data: the scale depends only on
    the block maximum, so scaling a block by 2^k leaves the codes unchanged and shifts e by
    k; negation flips only the sign bits."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    c0, s0 = oracle.quantize_rows(_bits(x), rule)
    for k in (-5, 1, 7):
        ck, sk = oracle.quantize_rows(_bits(np.ldexp(x, k)), rule)
        np.testing.assert_array_equal(ck, c0)
        np.testing.assert_array_equal(sk.astype(int), s0.astype(int) + k)
    cn, sn = oracle.quantize_rows(_bits(-x), rule)
    np.testing.assert_array_equal(cn, c0 ^ 0x88)
    np.testing.assert_array_equal(sn, s0)


def _grid_block_values(rng, shape, k):
    """Values g * 2^k with g on the E2M1 grid; element 0 of each 32-block is +-6 * 2^k."""
    g = rng.choice(np.concatenate([GRID, -GRID]), size=shape)
    g.reshape(-1, 32)[:, 0] = 6.0 * rng.choice([-1.0, 1.0], size=g.size // 32)
    return np.ldexp(g, k).astype(np.float32)


@pytest.mark.parametrize("rule", ["ocp", "uos"])
def test_quantize_grid_inputs_are_exact(rule):
    rng = np.random.default_rng(3)
    x = _grid_block_values(rng, (16, 128), -3)
    codes, scales = oracle.quantize_rows(_bits(x), rule)
    np.testing.assert_array_equal(oracle.dequantize_rows(codes, scales), x.astype(np.float64))
    assert np.all(scales == 127 - 3)


@pytest.mark.parametrize("N", [1, 31, 32, 100])
def test_quantize_cols_is_transposed_row_quantization(N):
    """V is quantized along tokens: column c of V, zero-padded to a multiple of 32, quantized as a row."""
    rng = np.random.default_rng(4)
    d = 64
    v = _bits(rng.standard_normal((2, N, d)).astype(np.float32) * 3)
    vc, vs = oracle.quantize_cols(v, "uos")
    npad = (N + 31) // 32 * 32
    for bh in range(2):
        vt = np.zeros((d, npad), dtype=np.uint16)
        vt[:, :N] = v[bh].T
        rc, rs = oracle.quantize_rows(vt, "uos")
        np.testing.assert_array_equal(vc[bh], rc)
        np.testing.assert_array_equal(vs[bh], rs)


# ----------------------------------------------------------------------------- attention loop


def _direct_softmax_attention(Q, K, V, scale):
    """Textbook softmax(Q K^T * scale) V in fp64 from bf16 values, two passes."""
    q = wl.bf16_bits_to_f32(Q).astype(np.float64)
    k = wl.bf16_bits_to_f32(K).astype(np.float64)
    v = wl.bf16_bits_to_f32(V).astype(np.float64)
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    p = np.exp(s - s.max(axis=-1, keepdims=True))
    return np.einsum("bhij,bhjd->bhid", p, v) / p.sum(axis=-1)[..., None]


@pytest.mark.parametrize("N,T", [(100, 32), (257, 64), (300, 128), (64, 64)])
def test_online_softmax_loop_equals_direct_softmax(N, T):
    Q, K, V = wl.gaussian_qkv(1, 2, N, 64, seed=5)
    scale = 1 / 8
    got = oracle.attention(Q, K, V, T, rule="none", pnq=True, scale=scale)
    ref = _direct_softmax_attention(Q, K, V, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("rule", ["ocp", "uos"])
@pytest.mark.parametrize("T", [64, 128])
def test_pnq_preserves_normalization_by_construction(rule, T):
    """With V = 1 everywhere, O = sum of the effective weights.  PNQ builds the row
    sum from the same quantized exponentials that weight V, so O == 1; without PNQ
    the row sum comes from unquantized values and O != 1 in general."""
    N, d = 300, 64
    Q, K, _ = wl.gaussian_qkv(1, 1, N, d, seed=6)
    Q = _bits(wl.bf16_bits_to_f32(Q) * 3)  # sharpen the softmax so P spans several binades
    ones = np.full((1, 1, N, d), 0x3F80, dtype=np.uint16)
    on = oracle.attention(Q, K, ones, T, rule=rule, pnq=True)
    np.testing.assert_allclose(on, 1.0, rtol=0, atol=1e-12)
    off = oracle.attention(Q, K, ones, T, rule=rule, pnq=False)
    assert np.max(np.abs(off - 1.0)) > 1e-3


@pytest.mark.parametrize("rule", ["ocp", "uos"])
@pytest.mark.parametrize("pnq", [True, False])
def test_zero_keys_give_mean_of_quantized_values(rule, pnq):
    """K = 0: every score is 0, every exponential is exactly 1 (code 4 with e = -2
    under both rules), so O is the column mean of the dequantized V."""
    N, d = 100, 64
    Q, _, V = wl.gaussian_qkv(1, 1, N, d, seed=7)
    K = np.zeros_like(Q)
    got = oracle.attention(Q, K, V, 64, rule=rule, pnq=pnq)
    vc, vs = oracle.quantize_cols(V, rule)
    vdq = oracle.dequantize_rows(vc, vs)[0, 0][:, :N]  # [d, N]
    np.testing.assert_allclose(got[0, 0], np.broadcast_to(vdq.mean(axis=1), (N, d)), rtol=1e-13, atol=1e-14)


def test_single_key_returns_its_quantized_value():
    Q, K, V = wl.gaussian_qkv(1, 1, 1, 64, seed=8)
    for rule in ("ocp", "uos"):
        got = oracle.attention(Q, K, V, 64, rule=rule, pnq=True)
        vc, vs = oracle.quantize_cols(V, rule)
        np.testing.assert_array_equal(got[0, 0, 0], oracle.dequantize_rows(vc, vs)[0, 0][:, 0])


def test_grid_inputs_make_input_quantization_exact():
    rng = np.random.default_rng(9)
    N, d = 96, 64
    q = _grid_block_values(rng, (1, 1, N, d), -2)
    k = _grid_block_values(rng, (1, 1, N, d), -3)
    vt = _grid_block_values(rng, (d, N), -1)  # 32-token blocks of each channel
    Q, K, V = _bits(q), _bits(k), _bits(vt.T[None, None].copy())
    for rule in ("ocp", "uos"):
        a = oracle.attention(Q, K, V, 32, rule=rule, pnq=True)
        b = oracle.attention(Q, K, V, 32, rule="none", p_rule=rule, pnq=True)
        np.testing.assert_array_equal(a, b)


def _two_key_case(N, kv_tile, scale, k_first):
    """Q row 0 = e_0; K rows given by their channel-0 value; V rows 0..N-2 = e_0, row N-1 = e_1."""
    d = 32
    q = np.zeros((1, 1, N, d), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, N, d), np.float32)
    k[0, 0, :, 0] = k_first
    v = np.zeros((1, 1, N, d), np.float32)
    v[0, 0, :-1, 0] = 1.0
    v[0, 0, -1, 1] = 1.0
    return _bits(q), _bits(k), _bits(v), scale


def test_hand_case_p_quantized_below_the_row_max():
    """Two keys, scores 0 and -1.5: exponentials 1 and e^-1.5 = 0.2231.  Block max 1
    gives e = -2 under both rules, e^-1.5 * 4 = 0.8925 rounds to 1.0, so the
    quantized weight is 0.25.  PNQ: O = (1, 0.25) / 1.25.  Without PNQ the row
    sum keeps the exact 0.2231: O = (1, 0.25) / 1.2231."""
    kf = np.array([0.0, -1.5], np.float32)
    Q, K, V, scale = _two_key_case(2, 32, 1.0, kf)
    p1 = math.exp(-1.5)
    for rule in ("ocp", "uos"):
        on = oracle.attention(Q, K, V, 32, rule=rule, pnq=True, scale=scale)[0, 0, 0, :2]
        np.testing.assert_allclose(on, [1 / 1.25, 0.25 / 1.25], rtol=1e-15)
        off = oracle.attention(Q, K, V, 32, rule=rule, pnq=False, scale=scale)[0, 0, 0, :2]
        np.testing.assert_allclose(off, [1 / (1 + p1), 0.25 / (1 + p1)], rtol=1e-15)


def test_hand_case_uos_versus_ocp_on_a_block_below_the_max():
    """Keys 0..31 score 0 (block 0 of the tile: 32 exponentials equal to 1); key 32
    alone in block 1 with exponential 0.95.  OCP: e = floor(log2 0.95) - 2 = -3,
    0.95 * 8 = 7.6 clips to 6, weight 0.75.  UOS: smallest e with 0.95 <= 7.25 * 2^e
    is -2, 0.95 * 4 = 3.8 rounds to 4, weight 1.0 -- the clipping side of the
    clipping-underflow trade-off the abstract names."""
    c = -math.log(0.95)
    kf = np.zeros(33, np.float32)
    kf[32] = -1.0
    Q, K, V, _ = _two_key_case(33, 64, c, kf)
    p = math.exp(-c)
    for rule, w in (("ocp", 0.75), ("uos", 1.0)):
        on = oracle.attention(Q, K, V, 64, rule=rule, pnq=True, scale=c)[0, 0, 0, :2]
        np.testing.assert_allclose(on, [32 / (32 + w), w / (32 + w)], rtol=1e-15)
        off = oracle.attention(Q, K, V, 64, rule=rule, pnq=False, scale=c)[0, 0, 0, :2]
        np.testing.assert_allclose(off, [32 / (32 + p), w / (32 + p)], rtol=1e-14)


def test_rows_subset_matches_full():
    Q, K, V = wl.gaussian_qkv(1, 2, 200, 64, seed=10)
    full = oracle.attention(Q, K, V, 64, rule="uos", pnq=True)
    rows = np.array([0, 63, 64, 199])
    sub = oracle.attention(Q, K, V, 64, rule="uos", pnq=True, rows=rows)
    np.testing.assert_array_equal(sub, full[:, :, rows])


def test_quality_direction_report(capsys):
    """Not a pin: error against exact attention for OCP without PNQ and for UOS
    with PNQ on small outlier inputs (the abstract claims the latter is closer)."""
    Q, K, V = wl.outlier_qkv(1, 2, 256, 128, seed=0)
    exact = oracle.attention(Q, K, V, 128, rule="none")
    errs = {}
    for rule, pnq in (("ocp", False), ("uos", True)):
        o = oracle.attention(Q, K, V, 128, rule=rule, pnq=pnq)
        errs[(rule, pnq)] = float(np.linalg.norm(o - exact) / np.linalg.norm(exact))
    with capsys.disabled():
        print(f"\n[quality] rel-Frobenius error vs exact: OCP/no-PNQ {errs[('ocp', False)]:.4e}, "
              f"UOS+PNQ {errs[('uos', True)]:.4e}")
    assert all(np.isfinite(list(errs.values())))
