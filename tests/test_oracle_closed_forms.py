"""Pins for the oracle's closed forms (F, Delta_c, delta_k, d_p) and the
bit-exact scaling claim, against textbook values and the E4M3 grid."""
import math

import numpy as np
import pytest

import oracle
from conftest import golden_facts

FACTS = golden_facts()


def grid():
    v = oracle.e4m3_decode(np.arange(128, dtype=np.uint8))
    return v[~np.isnan(v)]


def test_delta_k_textbook_values():
    # E[max of 2 standard normals] = 1/sqrt(pi); of 3 = 3/(2 sqrt(pi)).
    assert oracle.delta_k(1) == pytest.approx(0.0, abs=1e-10)
    assert oracle.delta_k(2) == pytest.approx(1 / math.sqrt(math.pi), abs=1e-9)
    assert oracle.delta_k(3) == pytest.approx(1.5 / math.sqrt(math.pi), abs=1e-9)
    # Monte Carlo for k = 4, and the pages' "about 1.0"
    rng = np.random.default_rng(0)
    mc = rng.standard_normal((2_000_000, 4)).max(1).mean()
    assert oracle.delta_k(4) == pytest.approx(mc, abs=3e-3)
    assert oracle.delta_k(4) == pytest.approx(FACTS["delta_k_for_k4"], abs=0.05)


def test_ten_ln2_is_the_printed_threshold():
    assert oracle.LN2_TEN == pytest.approx(FACTS["ln_threshold"], abs=5e-3)
    assert math.exp(-oracle.LN2_TEN) == pytest.approx(FACTS["e4m3_round_to_zero_threshold"], rel=1e-12)


def test_f_forward_is_a_normal_cdf_in_delta():
    # F(Delta_c(S), S) = 1/2 and F is Phi shifted by ln S.
    for S in [1.0, 4.0, 256.0, 448.0]:
        assert oracle.f_forward(oracle.delta_c(S), S) == pytest.approx(0.5, abs=1e-12)
    assert oracle.f_forward(5.0, 4.0) == pytest.approx(oracle.f_forward(5.0 - math.log(4.0), 1.0))
    # onset around Delta ~ 6-7 at S = 1 (the pages' wording): Delta_c(1) sits just below,
    # and F climbs from below 1/2 to above 1/2 across that band.
    assert 5.5 < oracle.delta_c(1.0) < FACTS["collapse_onset_high"]
    assert oracle.f_forward(FACTS["collapse_onset_low"], 1.0) > 0.5
    assert oracle.f_forward(4.0, 1.0) < 0.05


def test_f_row_reduces_to_plug_in_for_constant_rows():
    m = np.full(1000, 7.0 + oracle.delta_k(4))
    assert oracle.f_row(m, np.ones_like(m), 1.0) == pytest.approx(float(oracle.f_forward(7.0, 1.0)))


def test_dp_closed_form_matches_grid_brute_force():
    g = grid()
    for S in [2.0 ** e for e in range(-5, 9)] + [448.0, 3.0, 6.0, 12.0, 100.0, 300.0, 320.0, 384.0, 415.0]:
        assert oracle.dp_closed_form(S) == pytest.approx(oracle.dp_from_grid(S, g), rel=1e-12), S


def test_dp_printed_values():
    g = grid()
    for k in range(0, 9):
        assert oracle.dp_from_grid(2.0 ** k, g) == FACTS["dp_power_of_two"]
    excess = oracle.dp_from_grid(448.0, g) / oracle.dp_from_grid(256.0, g) - 1.0
    assert excess == pytest.approx(FACTS["dp_448_excess"], abs=0.005)
    # sawtooth: every scale between powers of two sits strictly above 2^-4 and below 2^-3
    for S in np.linspace(1.01, 447.0, 500):
        if math.log2(S) % 1 != 0:
            assert 2.0 ** -4 < oracle.dp_from_grid(S, g) < 2.0 ** -3


def test_normal_coverage_of_s256():
    # With S = 256, P * S stays in the E4M3 normal range for P down to 2^-6 / 256.
    min_normal = FACTS["e4m3_min_normal"]
    assert min_normal / 256.0 == FACTS["normal_coverage_s256"]
    g = grid()
    # smallest value whose gap to its lower neighbour is at most 1/8 of itself (3 mantissa bits)
    assert min(x for x in g if x > 0 and (x - max(y for y in g if y < x)) <= x / 8) == min_normal
    # 256 is the largest power of two not above the largest finite value
    assert max(2.0 ** e for e in range(16) if 2.0 ** e <= FACTS["e4m3_max_finite"]) == 256.0


def test_power_of_two_scaling_is_bit_exact_in_fp32():
    rng = np.random.default_rng(11)
    p = rng.random(1_000_000, dtype=np.float32)
    p = p[p > 0]
    for k in range(0, 9):
        S = np.float32(2.0 ** k)
        assert np.count_nonzero((p * S) / S != p) == 0
    S = np.float32(448.0)
    assert np.count_nonzero((p * S) / S != p) > 10_000
