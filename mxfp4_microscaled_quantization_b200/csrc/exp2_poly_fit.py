"""Derive the polynomial used for 2^f, f in [-1/2, 1/2], by the attention
kernel's FMA-pipe exponential (csrc/attention.cu, exp2_fma_x2).

Method (Cody & Waite style range reduction, "Software Manual for the
Elementary Functions", 1980): 2^w = 2^n * 2^f with n = round(w) and
f = w - n in [-1/2, 1/2]; 2^n is applied by adding n to the exponent field,
and 2^f comes from a degree-5 polynomial.  The polynomial here is a weighted
least-squares fit of 2^f on 400 Chebyshev nodes of [-1/2, 1/2] with weight
2^-f (so the fit minimises relative error), converted to monomial
coefficients and rounded to fp32.  Running this script prints the
coefficients and the maximum relative error of fp32 Horner evaluation on a
dense grid; the kernel's constants must equal the printed ones.
"""
import numpy as np
from numpy.polynomial import chebyshev as cheb

DEGREE = 5


def coefficients(degree=DEGREE):
    nodes = 0.5 * np.cos((2 * np.arange(400) + 1) / 800 * np.pi)
    c = cheb.chebfit(nodes, 2.0 ** nodes, degree, w=2.0 ** -nodes)
    return cheb.cheb2poly(c).astype(np.float32)


def horner_f32(coef, x):
    x = np.asarray(x, dtype=np.float32)
    p = np.full_like(x, coef[-1])
    for k in range(len(coef) - 2, -1, -1):
        p = (p * x + coef[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    coef = coefficients()
    f = np.linspace(-0.5, 0.5, 400001)
    rel = np.max(np.abs(horner_f32(coef, f).astype(np.float64) / 2.0 ** f - 1))
    for k, v in enumerate(coef):
        print(f"c{k} = {float(v).hex()}  ({float(v)!r})")
    print(f"max relative error (fp32 Horner) = {rel:.3e}")
