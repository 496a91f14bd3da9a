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
