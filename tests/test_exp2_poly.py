"""The attention kernel's FMA-pipe stand-ins for the MUFU exponential and its
log-domain block exponent of P, emulated in fp32 on the CPU.

- The exponential used without PNQ: its polynomial constants are the ones
  csrc/exp2_poly_fit.py derives (weighted Chebyshev least squares of 2^f on
  [-1/2, 1/2], degree 5), and fp32 Horner evaluation of them stays within
  2.5e-7 relative error of 2^f, on par with ex2.approx.
- The code-only stand-in used under PNQ (csrc/exp2_code_fit.py): a degree-6
  polynomial in u = sat((w + 2) / 8) whose E2M1 code equals that of 2^w except
  within fp32 rounding of a rounding point.
- The block exponent of P from the log2 of the block maximum: equal to the
  scale rule applied to the exact power of two except within fp32 rounding
  of a boundary."""
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
    """The stand-in's constants as written in csrc/ptx.cuh (c6 first), returned as c0 .. c6."""
    src = open(os.path.join(PKG, "csrc", "ptx.cuh")).read()
    body = src[src.index("void exp2_code_sat_x2("):]
    body = body[: body.index("v0 = __uint_as_float")]
    vals = [float.fromhex(h[:-1]) for h in re.findall(r"-?0x1\.[0-9a-f]+p[+-]\d+f", body)]
    return np.array(vals[::-1], dtype=np.float32)


def test_code_stand_in_uses_the_derived_coefficients():
    np.testing.assert_array_equal(_code_kernel_constants(), _code_fit_module().coefficients())


def test_code_stand_in_polynomial_shape():
    """p(0) = 0.25 exactly, p increasing on [0, 1] in fp32 evaluation, p(1) above
    the last rounding point 5, and p(u_t) = t to fp32 accuracy at each rounding
    point t, u_t = (log2 t + 2) / 8 (evaluated here in fp64, apart from the fit)."""
    m = _code_fit_module()
    coef = m.coefficients()
    u = np.linspace(0.0, 1.0, 400001, dtype=np.float64)
    p = m.stand_in_f32(coef, (u * 8.0 - 2.0).astype(np.float32)).astype(np.float64)
    assert p[0] == 0.25 and np.all(np.diff(p) >= 0) and p[-1] > 5.0
    for t in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
        uk = (np.log2(t) + 2.0) / 8.0
        val = sum(float(c) * uk ** i for i, c in enumerate(coef))
        assert abs(val / t - 1) < 2e-6, (t, val)


def test_code_stand_in_crossings_exact_fma():
    """With every FMA rounded once (exact rational emulation), at most 4 fp32 w
    within 64 ulp of each crossing log2 t land on the other side of t than 2^w,
    all within 2e-7 of the crossing."""
    m = _code_fit_module()
    for n, far in m.crossing_mismatches(m.coefficients(), ulps=64):
        assert n <= 4 and far <= 2e-7, (n, far)


def test_code_stand_in_gives_the_e2m1_code_of_2_pow_w():
    """The E2M1 code (round to nearest even, saturating) of the stand-in equals
    the code of the exact 2^w for every w on a dense grid over the range the
    kernel feeds it (w <= log2(8) after division by the block scale), apart from
    w within fp32 rounding of w + 2 (the stand-in's input is u = (w + 2) / 8) of
    a rounding point's crossing."""
    import oracle

    m = _code_fit_module()
    w = np.concatenate([np.linspace(-130.0, 3.0, 1_000_001), np.arange(-130, 4), [-np.inf]]).astype(np.float32)
    got = oracle.e2m1_encode(m.stand_in_f32(m.coefficients(), w).astype(np.float64))
    ref = oracle.e2m1_encode(2.0 ** w.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    crossings = np.log2([0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    for i in bad:
        tol = 2 * np.spacing(np.float32(np.float64(w[i]) + 2.0))
        assert np.min(np.abs(np.float64(w[i]) - crossings)) <= tol, w[i]
    assert len(bad) <= 12
    # every w below -2 is code 0; the tie at 2^-2 rounds to 0 as for the exact value
    assert np.all(got[w < -2] == 0) and got[w == -2][0] == 0
    # above the last crossing the code is the saturated 6 (code 7)
    assert np.all(got[w > np.log2(5.0) + 1e-6] == 7)


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
