"""The attention kernel's decisions on P, run through its own device functions
(mxattn_p_selftest) and compared with the CPU oracle.

MXAttention abstract ("MXAttention: Data-Free Optimal Scaling and
Pre-Normalization Quantization for MXFP4 Attention"): PNQ quantizes the
unnormalized exponentials to MXFP4.  The kernel decides each element's E2M1
code from 2^w in fp32 on one of three paths (ex2.approx, the FMA-pipe
code-only stand-in, the FMA-pipe degree-5 exponential) and each block's scale
in the log domain; the oracle decides from exact exponentials in fp64.  They
may differ only where the exact value lies within fp32 rounding of a decision
boundary, and the tests below check that on dense inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_microscaled_quantization_b200 import mxattn as mx

pytestmark = pytest.mark.gpu

E2M1_POINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])  # E2M1 rounding points (midpoints of the grid)


def _pad8(x):
    x = np.asarray(x, dtype=np.float32)
    return np.concatenate([x, np.full((-len(x)) % 8, x[-1], np.float32)])


def _run(path, x, qmax=7.25):
    out = mx.mxattn_p_selftest(path, torch.from_numpy(x).cuda(), qmax)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _near(x, points, width):
    """Inputs within `width` fp32 ulp of one of `points`, plus a dense grid."""
    parts = []
    for p in np.asarray(points, dtype=np.float64):
        c = np.float32(p)
        parts.append(c + np.arange(-width, width + 1, dtype=np.float32) * np.spacing(np.abs(c) + np.float32(1e-30)))
    return np.concatenate([x] + parts).astype(np.float32)


@pytest.mark.parametrize("path", [0, 1, 2])
def test_element_codes_of_exponentials(path):
    """Codes of 2^w over w in [-12, 3.2] (2^21 points) and every fp32 w within
    64 ulp of each rounding point's log2: equal to the exact value's code except
    within 1e-6 (log2 units) of a rounding point."""
    crossings = np.log2(E2M1_POINTS)
    w = _pad8(_near(np.linspace(-12.0, 3.2, 1 << 21, dtype=np.float64), crossings, 64))
    w = np.concatenate([w, _pad8([-np.inf, -1e4, -130.0, -2.0, 0.0, 2.5849625, 3.0, -126.5])])
    got = _run(path, w)
    ref = oracle.e2m1_encode(2.0 ** w.astype(np.float64))
    bad = np.nonzero(got != ref)[0]
    dist = np.min(np.abs(w[bad, None].astype(np.float64) - crossings[None, :]), axis=1) if len(bad) else np.zeros(0)
    assert np.all(dist <= 1e-6), w[bad][dist > 1e-6][:8]
    assert len(bad) <= 64, len(bad)
    print(f"[p-path {path}] {len(bad)} of {len(w)} codes differ, all within {dist.max() if len(bad) else 0:.1e} of a rounding point")


@pytest.mark.parametrize("qmax", [8.0, 7.25, 6.0, 4.5])
def test_mxfp4_block_exponent(qmax):
    """The log-domain block exponent against the oracle's scale rule on 2^x:
    identical except where x - log2(Qmax) lies within fp32 rounding (a few ulp
    of x) of an integer; never for OCP, whose boundaries are the integers
    themselves and are decided exactly."""
    L = 3.0 if qmax == 8.0 else np.log2(qmax)
    ints = np.arange(-140, 1, dtype=np.float64)
    x = _near(np.linspace(-140.0, 0.0, 1 << 20, dtype=np.float64), np.concatenate([ints + L - 3.0 * (qmax == 8.0), ints]), 8)
    # (0 > x > -1e-9 is left out: there 2^x rounds to 1 in fp64, while the kernel's floor(x) is exact)
    x = _pad8(np.concatenate([x[(x == 0) | (x < -1e-9)], np.float32([0.0, -0.0, -np.inf])]))
    got = _run(3, x, qmax)
    rule = "ocp" if qmax == 8.0 else qmax
    ref = oracle.scale_exponent(2.0 ** x.astype(np.float64), rule)
    bad = np.nonzero(got != ref)[0]
    if qmax == 8.0:
        assert len(bad) == 0, x[bad][:8]
    else:
        # fp32 rounding of log2(Qmax) - x is a few ulp of its magnitude (3.8e-6 at 40)
        frac = np.abs(x[bad].astype(np.float64) - L - np.round(x[bad].astype(np.float64) - L))
        tol = 4 * np.spacing(np.abs(x[bad]) + np.float32(L))
        assert np.all((frac <= tol) | (x[bad] < -125)), x[bad][frac > tol][:8]
        assert len(bad) <= 64


def test_nvfp4_block_scale():
    """The NVFP4 block scale E4M3(2^x * 448) against the oracle's E4M3 rounding
    of the exact product: identical except within 1e-6 (relative) of an E4M3
    rounding point."""
    x = _pad8(np.linspace(-30.0, 0.0, 1 << 21, dtype=np.float64))
    got = _run(4, x)
    exact = 2.0 ** x.astype(np.float64) * 448.0
    ref = oracle.e4m3_encode(exact)
    bad = np.nonzero(got != ref)[0]
    vals = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    rel = np.min(np.abs(exact[bad, None] / mids[None, :] - 1), axis=1) if len(bad) else np.zeros(0)
    assert np.all(rel <= 1e-6), x[bad][rel > 1e-6][:8]
    assert len(bad) <= 64


def test_e2m1_rounding_of_every_finite_fp32():
    """The rounding step alone (cvt.rn.satfinite.e2m1x2) on all 2^32 - 2^24 finite
    fp32 patterns, in chunks on the GPU: over the positive patterns the code never
    decreases and changes exactly 7 times, at the patterns the oracle's
    round-to-nearest-even rule puts them (just above 0.25, at 0.75, just above
    1.25, at 1.75, just above 2.5, at 3.5, just above 5); each negative pattern's
    code is the positive one's with the sign bit (-0 gives 0x8).  Since the
    oracle's rule is monotone with those same transitions, the two agree on
    every finite fp32 value."""
    transitions = []
    chunk = 1 << 27
    finite = 0x7F800000  # positive finite patterns: [0, 0x7F800000)
    prev = None
    for sign in (0, 1):
        for start in range(0, finite, chunk):
            stop = min(finite, start + chunk)
            bits = torch.arange(start, stop, dtype=torch.int64, device="cuda")
            if sign:
                bits = bits | (1 << 31)
            x = (bits - (1 << 32) * (bits >= (1 << 31))).to(torch.int32).view(torch.float32)
            n = x.numel() - x.numel() % 8
            codes = mx.mxattn_p_selftest(5, x[:n].contiguous())
            mag = codes & 7
            assert int((codes >> 3).min()) == sign and int((codes >> 3).max()) == sign
            d = mag[1:] - mag[:-1]
            assert bool((d >= 0).all())
            idx = torch.nonzero(d).flatten()
            for i in idx.tolist():
                transitions.append((sign, start + i + 1, int(mag[i]), int(mag[i + 1])))
            if prev is not None and prev[0] == sign and n:
                assert int(mag[0]) >= prev[1]
                if int(mag[0]) != prev[1]:
                    transitions.append((sign, start, prev[1], int(mag[0])))
            prev = (sign, int(mag[n - 1])) if n else prev
            # the few patterns left over by the multiple-of-8 cut
            del bits, x, codes, mag, d
    torch.cuda.synchronize()
    f = lambda b: float(np.array([b], dtype=np.uint32).view(np.float32)[0])  # noqa: E731
    pos = [(p, a, b) for s, p, a, b in transitions if s == 0]
    neg = [(p, a, b) for s, p, a, b in transitions if s == 1]
    assert [(a, b) for _, a, b in pos] == [(i, i + 1) for i in range(7)]
    assert [(a, b) for _, a, b in neg] == [(i, i + 1) for i in range(7)]
    for p, a, b in pos:
        v, below = f(p), f(p - 1)
        assert oracle.e2m1_encode([v])[0] == b and oracle.e2m1_encode([below])[0] == a, (v, below)
    assert [p for p, _, _ in neg] == [p for p, _, _ in pos]
