"""Pins of the oracle's GELU step (exact GELU v * Phi(v), fp64, then bf16), the
activation that the fused up-projection epilogue quantizes for the down projection.

What fixes it independently of the oracle's own formula:
  * textbook values of the standard normal CDF Phi at 1, 2, 3 (tables of Phi,
    e.g. Phi(1) = 0.841344746068543), giving GELU(v) = v * Phi(v) at +-1, +-2, +-3;
  * the identity GELU(v) - GELU(-v) = v (Phi(v) + Phi(-v) = 1), which a dropped
    term, a wrong sign or a swapped erf/erfc breaks;
  * the limits GELU(v) -> v for large v and -> -0 (relative accuracy kept) for very
    negative v, where the plain 1 + erf form cancels to zero;
  * the bf16 rounding of the result (the oracle's bf16 rounding is pinned in
    test_oracle_formats.py) and the ambiguity flag on constructed midpoints.
"""
import math

import numpy as np
import pytest

import oracle

# Phi(v) for v = 1, 2, 3 from standard normal tables (15 significant digits).
PHI = {1.0: 0.841344746068543, 2.0: 0.977249868051821, 3.0: 0.998650101968370}


@pytest.mark.parametrize("v", [1.0, 2.0, 3.0])
def test_textbook_values(v):
    assert oracle.gelu(v) == pytest.approx(v * PHI[v], rel=1e-14)
    assert oracle.gelu(-v) == pytest.approx(-v * (1.0 - PHI[v]), rel=1e-12)


def test_odd_part_identity():
    for v in np.linspace(-9.0, 9.0, 181):
        assert oracle.gelu(v) - oracle.gelu(-v) == pytest.approx(v, rel=1e-14, abs=1e-300)


def test_zero_and_limits():
    assert oracle.gelu(0.0) == 0.0
    assert oracle.gelu(12.0) == 12.0                       # Phi(12) rounds to 1 in fp64
    # deep negative tail: v * Phi(v) with Phi(v) ~ phi(v) / |v| (Mills ratio), not 0
    v = -20.0
    tail = v * math.exp(-v * v / 2) / math.sqrt(2 * math.pi) / abs(v) * (1 - 1 / v**2 + 3 / v**4)
    assert oracle.gelu(v) == pytest.approx(tail, rel=1e-4)
    assert oracle.gelu(v) < 0.0


def _bf16_bits(values):
    return oracle.bf16_from_double(np.asarray(values, dtype=np.float64))


def test_bf16_output_matches_rounded_fp64_value():
    y = _bf16_bits([-6.0, -1.5, -0.25, 0.0, 0.125, 0.75, 1.0, 3.5, 100.0])
    h, amb = oracle.gelu_bf16(y)
    vals = oracle.bf16_bits_to_f64(y)
    want = _bf16_bits([oracle.gelu(v) for v in vals])
    assert np.array_equal(h, want)
    assert h[3] == 0 and not amb[3]            # GELU(0) = +0 exactly
    assert oracle.bf16_bits_to_f64(h[-1:])[0] == 100.0


def test_ambiguity_band_grows_with_v_squared():
    # with only the v^2 term, the flag is set exactly where the fp64 GELU lies within
    # sq * v^2 * |GELU| of the midpoint of its two bf16 neighbours
    sq = 2.0 ** -16
    y = np.arange(0x3E00, 0x4100, dtype=np.uint16)  # 0.125 .. 8 in bf16
    h, amb = oracle.gelu_bf16(y, rel_tol=0.0, rel_tol_sq=sq)
    v = oracle.bf16_bits_to_f64(y)
    g = np.array([oracle.gelu(t) for t in v])
    hv = oracle.bf16_bits_to_f64(h)
    other = np.where(g > hv, h + 1, h - 1).astype(np.uint16)
    mid = 0.5 * (hv + oracle.bf16_bits_to_f64(other))
    want = (g != hv) & (np.abs(g - mid) <= sq * v * v * np.abs(g))
    assert np.array_equal(amb, want)
    assert amb.any()
    wider = oracle.gelu_bf16(y, rel_tol=0.0, rel_tol_sq=4 * sq)[1]
    assert np.all(wider[amb]) and wider.sum() > amb.sum()   # a wider band flags a superset
    assert not oracle.gelu_bf16(y, rel_tol=0.0, rel_tol_sq=0.0)[1].any()


def test_ambiguity_flag_marks_values_near_a_bf16_midpoint():
    # scan bf16 inputs; the flag must be set exactly where the fp64 GELU lies within
    # rel_tol of the midpoint of its two bf16 neighbours
    rel = 2.0 ** -12  # coarse tolerance so that the scan finds flagged values
    y = np.arange(0x3E00, 0x4100, dtype=np.uint16)  # 0.125 .. 8 in bf16
    h, amb = oracle.gelu_bf16(y, rel_tol=rel, rel_tol_sq=0.0)
    vals = oracle.bf16_bits_to_f64(y)
    g = np.array([oracle.gelu(v) for v in vals])
    hv = oracle.bf16_bits_to_f64(h)
    # neighbour on the other side of g (positive values: next / previous bit pattern)
    other = np.where(g > hv, h + 1, h - 1).astype(np.uint16)
    mid = 0.5 * (hv + oracle.bf16_bits_to_f64(other))
    want = (g != hv) & (np.abs(g - mid) <= rel * np.abs(g))
    assert np.array_equal(amb, want)
    assert amb.any() and not amb.all()
    # h is the nearer neighbour: never farther from g than the other one
    assert np.all(np.abs(g - hv) <= np.abs(g - oracle.bf16_bits_to_f64(other)))
