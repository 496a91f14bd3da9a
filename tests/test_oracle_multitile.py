"""Pins of the oracle's multi-tile softmax loop (CPU).

The abstract of "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
Quantization for MXFP4 Attention" places PNQ inside the softmax loop: the
unnormalized exponentials of each key tile are quantized before the row sum is
formed.  The oracle reads "unnormalized" as exp(s - m) with m the running row
maximum *after* the current tile (standard online softmax); a tile's quantized
values are afterwards only multiplied by the factors alpha = exp(m_old - m_new)
of later tiles.  The cases below have two key tiles and hand-derived outputs
that follow from that reading alone, so they fail for the two plausible
misreadings:

* quantizing exp(s - tile max) and carrying the factor exp(tile max - m_new)
  (caught by a tile whose own maximum lies below the running maximum);
* a two-pass form that quantizes every tile against the final row maximum
  (caught by a tile that precedes the row maximum).

Each misreading is also planted in a copy of the oracle's C source at test
time, compiled, and shown to fail the pin it targets.

Construction: d = 32, every query row is e_0, key j is k_j * e_0, so every
score is s_j = k_j * scale exactly (Q and K quantize exactly: their blocks
hold 0, 1 or -64).  V is one-hot: key j puts a 1 in channel group[j], which
also quantizes exactly, so O's first channels are sums of effective weights
divided by l.
"""
from __future__ import annotations

import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from mxfp4_microscaled_quantization_b200 import workloads as wl

T = 32
N = 64


def _bits(x):
    return wl.f32_to_bf16_bits(np.asarray(x, np.float32))


def _inputs(kvals, group, d=32):
    n = len(kvals)
    q = np.zeros((1, 1, n, d), np.float32)
    q[..., 0] = 1.0
    k = np.zeros((1, 1, n, d), np.float32)
    k[0, 0, :, 0] = kvals
    v = np.zeros((1, 1, n, d), np.float32)
    v[0, 0, np.arange(n), group] = 1.0
    return _bits(q), _bits(k), _bits(v)


def _case_max_in_second_tile():
    """Tile 0 (keys 0..31): score 0.  Tile 1: key 32 scores 1, keys 33..63 score -64.
    V: tile-0 keys -> channel 0, key 32 -> channel 1, keys 33..63 -> channel 2.  Scale 1."""
    kvals = [0.0] * 32 + [1.0] + [-64.0] * 31
    group = [0] * 32 + [1] + [2] * 31
    return _inputs(kvals, group), 1.0


def _case_max_in_first_tile():
    """Key 0 scores c, keys 1..63 score 0, with c = -ln 0.95, so every exponential
    other than key 0's is exp(-c) = 0.95 against the running maximum c.
    V: key 0 -> channel 0, keys 1..31 -> channel 1, keys 32..63 -> channel 2."""
    c = -math.log(0.95)
    kvals = [1.0] + [0.0] * 63
    group = [0] + [1] * 31 + [2] * 32
    return _inputs(kvals, group), c


def _expected_mxfp4_max_in_second_tile(pnq):
    """Tile 0 at m = 0: all 32 exponentials are 1; block maximum 1 gives e = -2 under
    both rules, 1 * 4 = 4 is an E2M1 value, so each quantized weight is exactly 1.
    Tile 1 raises m to 1 (alpha = e^-1): key 32's exponential is 1 (weight 1), the
    others are e^-65 and quantize to 0 (e^-65 * 4 < 0.25).  Tile 0's weights end as
    e^-1 each.  l (PNQ) = 32 e^-1 + 1; l (no PNQ) adds the unquantized 31 e^-65."""
    a = math.exp(-1.0)
    l = 32 * a + 1 + (0.0 if pnq else 31 * math.exp(-65.0))
    return np.array([32 * a, 1.0, 0.0]) / l


def _expected_mxfp4_max_in_first_tile(rule, pnq):
    """Tile 0 at m = c: block maximum 1 (key 0) gives e = -2; key 0 -> 4 (weight 1),
    keys 1..31: 0.95 * 4 = 3.8 rounds to 4 (weight 1).  Tile 1: its own maximum 0
    lies below m = c, so m stays c (alpha = 1) and its 32 exponentials are 0.95 each,
    quantized as a block with maximum 0.95:
      OCP: e = floor(log2 0.95) - 2 = -3, 0.95 * 8 = 7.6 saturates to 6 -> weight 0.75;
      UOS: smallest e with 0.95 <= 7.25 * 2^e is -2, 0.95 * 4 = 3.8 -> 4 -> weight 1.
    l (PNQ) = 32 + 32 w; l (no PNQ) = 1 + 63 * 0.95."""
    p = math.exp(-(-math.log(0.95)))
    w = 0.75 if rule == "ocp" else 1.0
    l = (32 + 32 * w) if pnq else (1 + 63 * p)
    return np.array([1.0, 31.0, 32 * w]) / l


# NVFP4 (reading: 16-key blocks of P with scale sb = E4M3(fp32(pmax) * 448) and
# element code E2M1(p * fp32(2688 / sb)), weight = code value * sb / 2688).
Q416 = 6.0 * 416.0 / 2688.0  # a block whose maximum exponential is 0.95: sb = E4M3(425.6) = 416, 0.95 * 6.46 -> 6


def _expected_nvfp4_max_in_second_tile(pnq):
    """As the MXFP4 case: exponentials of 1 give sb = 448 and code 6, weight exactly 1;
    the block of keys 48..63 has pmax = e^-65, its scale rounds to 0 and its weights
    are 0.  So the expected values equal the MXFP4 ones."""
    return _expected_mxfp4_max_in_second_tile(pnq)


def _expected_nvfp4_max_in_first_tile(pnq):
    """Tile 0: keys 0..15 (pmax 1, sb 448): key 0 -> 6 (weight 1), keys 1..15: 0.95 * 6
    = 5.7 -> 6 (weight 1); keys 16..31 (pmax 0.95, sb 416): weight Q416 each.  Tile 1
    (m unchanged, alpha = 1): two blocks with pmax 0.95, weight Q416 each."""
    p = 0.95
    if pnq:
        l = 16 + 48 * Q416
    else:
        l = 1 + 63 * math.exp(math.log(p))
    return np.array([1.0, 15 + 16 * Q416, 32 * Q416]) / l


def _o_mxfp4(inputs, scale, rule, pnq):
    Q, K, V = inputs
    return oracle.attention(Q, K, V, T, rule=rule, pnq=pnq, scale=scale)[0, 0]


def _o_nvfp4(inputs, scale, pnq):
    Q, K, V = inputs
    return oracle.nvfp4_attention(Q, K, V, T, pnq=pnq, scale=scale)[0, 0]


@pytest.mark.parametrize("rule", ["ocp", "uos"])
@pytest.mark.parametrize("pnq", [True, False])
def test_mxfp4_first_tile_quantized_at_its_own_running_max(rule, pnq):
    inputs, scale = _case_max_in_second_tile()
    o = _o_mxfp4(inputs, scale, rule, pnq)
    want = _expected_mxfp4_max_in_second_tile(pnq)
    np.testing.assert_allclose(o[:, :3], np.broadcast_to(want, (N, 3)), rtol=1e-14, atol=0)
    assert np.all(o[:, 3:] == 0)


@pytest.mark.parametrize("rule", ["ocp", "uos"])
@pytest.mark.parametrize("pnq", [True, False])
def test_mxfp4_later_tile_quantized_against_the_running_max(rule, pnq):
    inputs, scale = _case_max_in_first_tile()
    o = _o_mxfp4(inputs, scale, rule, pnq)
    want = _expected_mxfp4_max_in_first_tile(rule, pnq)
    np.testing.assert_allclose(o[:, :3], np.broadcast_to(want, (N, 3)), rtol=1e-14, atol=0)


@pytest.mark.parametrize("pnq", [True, False])
def test_nvfp4_first_tile_quantized_at_its_own_running_max(pnq):
    inputs, scale = _case_max_in_second_tile()
    o = _o_nvfp4(inputs, scale, pnq)
    want = _expected_nvfp4_max_in_second_tile(pnq)
    np.testing.assert_allclose(o[:, :3], np.broadcast_to(want, (N, 3)), rtol=1e-14, atol=0)


@pytest.mark.parametrize("pnq", [True, False])
def test_nvfp4_later_tile_quantized_against_the_running_max(pnq):
    inputs, scale = _case_max_in_first_tile()
    o = _o_nvfp4(inputs, scale, pnq)
    want = _expected_nvfp4_max_in_first_tile(pnq)
    np.testing.assert_allclose(o[:, :3], np.broadcast_to(want, (N, 3)), rtol=1e-14, atol=0)


def test_expected_values_separate_the_rules():
    """The later-tile case is a real UOS-versus-OCP case: the two expected outputs differ."""
    a = _expected_mxfp4_max_in_first_tile("ocp", True)
    b = _expected_mxfp4_max_in_first_tile("uos", True)
    assert np.max(np.abs(a - b)) > 1e-2


# ----------------------------------------------------------------------------- planted mistakes

def _replace(src: str, old: str, new: str, count: int) -> str:
    assert src.count(old) == count, (old, src.count(old))
    return src.replace(old, new)


def _mutant_tile_local(src: str) -> str:
    """Quantize exp(s - tile max) and carry exp(tile max - m_new) as a factor."""
    src = _replace(src, "exp(s[j] - m_new)", "exp(s[j] - tile_max)", 1)
    src = _replace(src, "exp(sc[j] - m_new)", "exp(sc[j] - tile_max)", 1)
    return _replace(src, "sum_p += p[k];",
                    "p[k] *= exp(tile_max - m_new); q[k] *= exp(tile_max - m_new); sum_p += p[k];", 2)


def _mutant_final_max(src: str) -> str:
    """Two passes: every tile quantized against the final row maximum, no rescaling."""
    for arr in ("s", "sc"):
        src = _replace(src, f"exp({arr}[j] - m_new)", f"exp({arr}[j] - row_max)", 1)
    src = _replace(src, "double m = -INFINITY, l = 0.0;",
                   "double row_max = -INFINITY; for (int64_t jj = 0; jj < N; jj++) "
                   "{ double sj = ROWSCORE[jj]; if (sj > row_max) row_max = sj; } double m = -INFINITY, l = 0.0;", 2)
    # the first occurrence is the MXFP4 loop (scores in s), the second the NVFP4 loop (scores in sc)
    src = src.replace("ROWSCORE", "s", 1).replace("ROWSCORE", "sc", 1)
    return _replace(src, "double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);",
                    "double alpha = (m == -INFINITY) ? 0.0 : 1.0;", 2)


def _build_mutant(tmp_path, mutate):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    c = tmp_path / "oracle_mutant.c"
    c.write_text(mutate(src))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                    "-o", str(so), str(c), "-lm"], check=True)
    return oracle.load(str(so))


@pytest.mark.parametrize("mutant,case", [(_mutant_tile_local, "first"), (_mutant_final_max, "second")])
def test_planted_misreadings_fail_the_pins(tmp_path, monkeypatch, mutant, case):
    """Each misreading, planted in a copy of the oracle, breaks the pin built for it,
    for both formats, both rules and PNQ on and off."""
    oracle.lib()  # make sure the real library is loaded before swapping it out
    lib = _build_mutant(tmp_path, mutant)
    monkeypatch.setattr(oracle, "_lib", lib)
    if case == "first":
        inputs, scale = _case_max_in_first_tile()
        for pnq in (True, False):
            for rule in ("ocp", "uos"):
                o = _o_mxfp4(inputs, scale, rule, pnq)[0, :3]
                assert not np.allclose(o, _expected_mxfp4_max_in_first_tile(rule, pnq), rtol=1e-6, atol=0)
            o = _o_nvfp4(inputs, scale, pnq)[0, :3]
            assert not np.allclose(o, _expected_nvfp4_max_in_first_tile(pnq), rtol=1e-6, atol=0)
    else:
        inputs, scale = _case_max_in_second_tile()
        for pnq in (True, False):
            for rule in ("ocp", "uos"):
                o = _o_mxfp4(inputs, scale, rule, pnq)[0, :3]
                assert not np.allclose(o, _expected_mxfp4_max_in_second_tile(pnq), rtol=1e-6, atol=0)
            o = _o_nvfp4(inputs, scale, pnq)[0, :3]
            assert not np.allclose(o, _expected_nvfp4_max_in_second_tile(pnq), rtol=1e-6, atol=0)
