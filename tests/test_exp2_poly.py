"""The FMA-pipe exponential of the attention kernel: its polynomial constants
are the ones csrc/exp2_poly_fit.py derives (weighted Chebyshev least squares
of 2^f on [-1/2, 1/2], degree 5), and fp32 Horner evaluation of them stays
within 2.5e-7 relative error of 2^f, on par with the MUFU ex2.approx."""
import importlib.util
import os
import re

import numpy as np

PKG = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "mxfp4_microscaled_quantization_b200")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit", os.path.join(PKG, "csrc", "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_constants():
    src = open(os.path.join(PKG, "csrc", "ptx.cuh")).read()
    body = src[src.index("void exp2_fma_x2("):]
    body = body[: body.index("v0 = __uint_as_float")]
    return np.array([float.fromhex(h[:-1]) for h in re.findall(r"0x1\.[0-9a-f]+p[+-]\d+f", body)], dtype=np.float32)


def test_kernel_uses_the_derived_coefficients():
    np.testing.assert_array_equal(_kernel_constants(), _fit_module().coefficients())


def test_polynomial_relative_error_bound():
    m = _fit_module()
    f = np.linspace(-0.5, 0.5, 200001)
    p = m.horner_f32(m.coefficients(), f).astype(np.float64)
    assert np.max(np.abs(p / 2.0 ** f - 1)) < 2.5e-7


def test_range_reduction_reconstructs_powers_of_two():
    """2^w = 2^round(w) * 2^(w - round(w)) over the clamped input range, emulated in fp32
    the way the kernel does it (round via adding 1.5 * 2^23, exponent via an integer add)."""
    m = _fit_module()
    coef = m.coefficients()
    w = np.concatenate([np.linspace(-125, 3, 100001), np.arange(-125, 4)]).astype(np.float32)
    c = np.float32(12582912.0)
    t = (w + c).astype(np.float32)
    n = (t - c).astype(np.float32)
    f = (w - n).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    p = m.horner_f32(coef, f)
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    v = bits.view(np.float32).astype(np.float64)
    assert np.max(np.abs(v / 2.0 ** w.astype(np.float64) - 1)) < 2.5e-7


# ---------------------------------------------------------------- code-only stand-in for 2^w (PNQ)

def _code_fit_module():
    spec = importlib.util.spec_from_file_location("exp2_code_fit", os.path.join(PKG, "csrc", "exp2_code_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _code_kernel_constants():
    src = open(os.path.join(PKG, "csrc", "ptx.cuh")).read()
    body = src[src.index("void exp2_code_x2("):]
    body = body[: body.index("v0 = __uint_as_float")]
    return np.array([float.fromhex(h[:-1]) for h in re.findall(r"0x1\.[0-9a-f]+p[+-]\d+f", body)], dtype=np.float32)


def _code_stand_in_f32(w):
    """exp2_code_x2 emulated in fp32 the way the kernel runs it: clamp at -8,
    floor via adding 1.5 * 2^23 rounded toward -inf, the cubic in Horner form,
    2^floor(w) added to the exponent field."""
    m = _code_fit_module()
    w = np.maximum(np.asarray(w, dtype=np.float32), np.float32(-8.0))
    c = np.float64(12582912.0)
    # fp32 add with round-toward-minus-infinity: the fp64 sum is exact here, floor it to the fp32 grid (ulp 1)
    t = np.floor(w.astype(np.float64) + c).astype(np.float32)
    n = (t - np.float32(c)).astype(np.float32)
    f = (w - n).astype(np.float32)
    z = m.horner_f32(m.coefficients(), f)
    bits = (z.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_code_stand_in_uses_the_derived_coefficients():
    np.testing.assert_array_equal(_code_kernel_constants(), _code_fit_module().coefficients())


def test_code_stand_in_cubic_shape():
    """z(0) = 1 exactly, increasing on [0, 1), below 2, and on the right side of
    each mantissa rounding point everywhere except a few ulp around it."""
    m = _code_fit_module()
    coef = m.coefficients()
    f = np.linspace(0.0, 1.0, 400001, dtype=np.float64).astype(np.float32)[:-1]
    z = m.horner_f32(coef, f).astype(np.float64)
    assert z[0] == 1.0 and np.all(np.diff(z) >= 0) and z.max() < 2.0
    assert all(k <= 4 for k in m.crossing_mismatches(coef, ulps=256))


def test_code_stand_in_gives_the_e2m1_code_of_2_pow_w():
    """The E2M1 code (round to nearest even, saturating) of the stand-in equals
    the code of the exact 2^w for every w on a dense grid over the range the
    kernel feeds it (w <= log2(8) after division by the block scale), apart from
    w within 4 fp32 ulp of a rounding point's crossing."""
    import oracle

    w = np.concatenate([np.linspace(-130.0, 3.0, 1_000_001), np.arange(-130, 4), [-np.inf]]).astype(np.float32)
    got = oracle.e2m1_encode(_code_stand_in_f32(w).astype(np.float64))
    exact = 2.0 ** w.astype(np.float64)
    ref = oracle.e2m1_encode(exact)
    bad = np.nonzero(got != ref)[0]
    crossings = np.log2([0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    for i in bad:
        assert np.min(np.abs(np.float64(w[i]) - crossings)) <= 4 * np.spacing(np.float32(abs(w[i]) + 1)), w[i]
    assert len(bad) <= 12
    # every w below -2 is code 0; the tie at 2^-2 rounds to 0 as for the exact value
    assert np.all(got[w < -2] == 0) and got[w == -2][0] == 0


# ---------------------------------------------------------------- block exponent of P in the log domain

def _log_domain_exponent(x, qmax):
    """The attention kernel's block exponent of P from x = log2 of the block's
    largest exponential, emulated in fp32: e = s * floor(s * x + off) + add with
    (s, off, add) = (-1, log2(Qmax), 0) for a boundary below 8 and (+1, 0, -2)
    for OCP."""
    x = np.asarray(x, dtype=np.float32)
    if qmax == 8.0:
        s, off, add = np.float32(1.0), np.float32(0.0), -2
    else:
        s, off, add = np.float32(-1.0), np.float32(np.log2(qmax)), 0
    z = (s * x + off).astype(np.float32)
    z = np.clip(z, np.float32(-250.0), np.float32(250.0))
    e = (s * np.floor(z)).astype(np.int64) + add
    return np.maximum(e, -127)


def test_log_domain_block_exponent_matches_the_scale_rule():
    """Against the oracle's scale rule applied to 2^x: identical for every x
    except within fp32 rounding of a boundary crossing (x - log2 Qmax an integer),
    and exact at integer x (the block holding the row maximum has x = 0)."""
    import oracle

    rng = np.random.default_rng(3)
    x = np.concatenate([-np.abs(rng.standard_normal(200_000)) * 40, -np.arange(0, 140), [0.0, -0.0, -1e-30]])
    x = x.astype(np.float32)
    for qmax, rule in [(8.0, "ocp"), (7.25, "uos"), (5.0, 5.0), (6.5, 6.5), (4.5, 4.5), (7.875, 7.875)]:
        got = _log_domain_exponent(x, qmax)
        ref = oracle.scale_exponent(2.0 ** x.astype(np.float64), rule).astype(np.int64)
        bad = np.nonzero(got != ref)[0]
        L = np.log2(qmax)
        for i in bad:  # only where x - log2 Qmax lies within fp32 rounding of an integer
            frac = np.float64(x[i]) - L - np.round(np.float64(x[i]) - L)
            assert abs(frac) <= 4 * np.spacing(np.float32(abs(x[i]) + L)), (qmax, x[i], got[i], ref[i])
        if qmax == 8.0:
            # floor(x) - 2 is exact in fp32; the one difference is x = -1e-30, where the
            # kernel's floor is right and 2^x in fp64 rounds up to the boundary 1.0
            assert list(x[bad]) == [np.float32(-1e-30)], x[bad[:5]]
        assert len(bad) <= 10
        assert np.all(got[x == 0] == ref[x == 0])
