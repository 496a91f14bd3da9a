"""Derive the cubic used by the attention kernel's code-only stand-in for 2^w
(csrc/ptx.cuh, exp2_code_x2), which puts part of the PNQ exponentials on the
FMA pipe.

Under PNQ only the E2M1 code of each exponential is kept (the row sum comes
from the tensor core), and the code of 2^w is fixed by where w falls against
the E2M1 rounding points.  With n = floor(w) and f = w - n in [0, 1), the
value 2^n * z(f) has the code of 2^w whenever z(0) = 1, z is increasing on
[0, 1), z < 2, and z crosses the mantissa rounding points 1.25, 1.5 and 1.75
where 2^f does, i.e. at f = log2(1.25), log2(1.5), log2(1.75):
  binade [1/4, 1/2): the tie at 1/4 sits at f = 0;
  binade [1/2, 1):   rounding point 3/4 = 1.5 / 2;
  binades [1, 2), [2, 4), [4, 8): points 1.25 and 1.75 times 2^n (and 6 and
  up saturate).
z(f) = 1 + c1 f + c2 f^2 + c3 f^3 is the cubic through those three points
(solved exactly in fp64, then rounded to fp32).  Running this script prints
the coefficients, checks monotonicity and z < 2 in fp32 Horner evaluation,
and counts fp32 values of f near each crossing point whose side differs from
that of 2^f; the kernel's constants must equal the printed ones.
"""
import numpy as np

POINTS = np.array([1.25, 1.5, 1.75])


def coefficients():
    f = np.log2(POINTS)
    a = np.stack([f, f ** 2, f ** 3], axis=1)
    return np.linalg.solve(a, POINTS - 1.0).astype(np.float32)  # c1, c2, c3


def horner_f32(coef, f):
    f = np.asarray(f, dtype=np.float32)
    c1, c2, c3 = (np.float32(c) for c in coef)
    p = np.full_like(f, c3)
    p = (p * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    return (p * f + np.float32(1.0)).astype(np.float32)


def crossing_mismatches(coef, ulps=64):
    """Per rounding point: fp32 f within `ulps` ulp of the crossing whose side
    (z(f) vs the point) differs from that of the exact 2^f."""
    out = []
    for t in POINTS:
        f0 = np.float32(np.log2(t))
        fs = (f0 + np.arange(-ulps, ulps + 1, dtype=np.float32) * np.spacing(f0)).astype(np.float32)
        z = horner_f32(coef, fs).astype(np.float64)
        out.append(int(np.sum((z >= t) != (2.0 ** fs.astype(np.float64) >= t))))
    return out


if __name__ == "__main__":
    coef = coefficients()
    for k, v in enumerate(coef, start=1):
        print(f"c{k} = {float(v).hex()}  ({float(v)!r})")
    f = np.linspace(0.0, 1.0, 1000001, dtype=np.float64).astype(np.float32)[:-1]
    z = horner_f32(coef, f).astype(np.float64)
    print("increasing:", bool(np.all(np.diff(z) >= 0)), " z(0) =", z[0], " max z =", z.max())
    print("max |z(f) - 2^f| =", float(np.max(np.abs(z - 2.0 ** f.astype(np.float64)))))
    print("side mismatches within 64 ulp of each crossing:", crossing_mismatches(coef))
