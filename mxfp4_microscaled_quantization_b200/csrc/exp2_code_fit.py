"""Derive the polynomial used by the attention kernel's code-only stand-in for
2^w (csrc/ptx.cuh, exp2_code_sat_x2), which puts part of the PNQ
exponentials on the FMA pipe.

Under PNQ only the E2M1 code of each exponential is kept (the row sum comes
from the tensor core), and the code of 2^w is fixed by where w falls against
the seven E2M1 rounding points 0.25, 0.75, 1.25, 1.75, 2.5, 3.5 and 5 (values
above 5 all round to 6 or saturate there; values at or below 0.25 give 0, the
tie at 0.25 going to the even code 0).  The stand-in maps w onto
u = sat((w + 2) / 8), clamped to [0, 1] by the saturating FMA that forms it
(w <= -2 gives u = 0), and evaluates a degree-6 polynomial p(u) with
  p(0) = 0.25 exactly (so w <= -2 keeps code 0, and w just above -2 gets 1),
  p((log2 t + 2) / 8) = t for the other six rounding points t,
  p increasing on [0, 1] (so p crosses each rounding point once, where 2^w
  does, and p(1) > 5 gives the saturated code for every w above log2 5).
Seven conditions fix the seven coefficients.  They are solved in fp64 and
rounded to fp32.  The kernel evaluates p with fp32 FMAs (Horner), so running
this script also checks, with the FMAs emulated exactly (fractions), that the
side of every rounding point on which p(u(w)) lands equals that of 2^w for all
fp32 w except a few next to each crossing.  The kernel's constants must equal
the printed ones.
"""
from fractions import Fraction

import numpy as np

POINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
W_LO, SPAN = -2.0, 8.0  # u = (w - W_LO) / SPAN; both scalings are exact in fp32


def coefficients():
    """c0 .. c6 as fp32 (c0 = 0.25)."""
    u = (np.log2(POINTS) - W_LO) / SPAN
    a = np.stack([u[1:] ** i for i in range(1, 7)], axis=1)
    c = np.linalg.solve(a, POINTS[1:] - POINTS[0])
    return np.concatenate([[POINTS[0]], c]).astype(np.float32)


def _round_f32(q: Fraction) -> np.float32:
    """Round a rational to the nearest fp32 (ties to even)."""
    x = np.float32(float(q))
    best = x
    for c in (np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(-np.inf))):
        dc, db = abs(Fraction(float(c)) - q), abs(Fraction(float(best)) - q)
        if dc < db or (dc == db and int(np.float32(c).view(np.uint32)) % 2 == 0):
            best = c
    return np.float32(best)


def fma_f32_exact(a, b, c) -> np.float32:
    return _round_f32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def stand_in_exact(coef, w) -> np.float32:
    """The kernel's arithmetic on one fp32 w, every FMA rounded once."""
    u = fma_f32_exact(np.float32(w), np.float32(1.0 / SPAN), np.float32(-W_LO / SPAN))
    u = min(max(u, np.float32(0.0)), np.float32(1.0))
    p = coef[6]
    for i in range(5, -1, -1):
        p = fma_f32_exact(p, u, coef[i])
    return p


def stand_in_f32(coef, w):
    """Vectorised version: fp64 products are exact, the sum is rounded to fp64
    and then to fp32, which can differ from one FMA rounding only when the fp64
    sum lands on an fp32 midpoint (a one-ulp difference, visible in the code only
    next to a rounding point)."""
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    u = np.clip((w * (1.0 / SPAN) + (-W_LO / SPAN)).astype(np.float32), 0.0, 1.0).astype(np.float64)
    p = np.full(u.shape, np.float64(coef[6]))
    for i in range(5, -1, -1):
        p = (p * u + np.float64(coef[i])).astype(np.float32).astype(np.float64)
    return p.astype(np.float32)


def crossing_mismatches(coef, ulps=64):
    """Per rounding point above 0.25: the fp32 w within `ulps` ulp of log2 t
    whose stand-in lands on the other side of t than 2^w does, and the largest
    |w - log2 t| among them."""
    out = []
    for t in POINTS[1:]:
        w0 = np.float32(np.log2(t))
        ws = [w0]
        for d in (np.float32(np.inf), np.float32(-np.inf)):
            x = w0
            for _ in range(ulps):
                x = np.nextafter(x, d)
                ws.append(x)
        bad = [w for w in ws if (Fraction(float(stand_in_exact(coef, w))) > Fraction(float(t)))
               != (float(w) > np.log2(t))]
        out.append((len(bad), max((abs(float(w) - np.log2(t)) for w in bad), default=0.0)))
    return out


if __name__ == "__main__":
    coef = coefficients()
    for k, v in enumerate(coef):
        print(f"c{k} = {float(v).hex()}  ({float(v)!r})")
    u = np.linspace(0.0, 1.0, 1000001, dtype=np.float64).astype(np.float32)
    p = stand_in_f32(coef, (u.astype(np.float64) * SPAN + W_LO).astype(np.float32)).astype(np.float64)
    print("increasing:", bool(np.all(np.diff(p) >= 0)), " p(0) =", p[0], " p(1) =", p[-1])
    print("per rounding point (wrong-side w within 64 ulp, farthest |w - log2 t|):", crossing_mismatches(coef))
