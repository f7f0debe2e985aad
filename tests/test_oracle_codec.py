"""Pins for the oracle's E4M3 codec and bfloat16 rounding.

The codec is pinned to things other than itself: PyTorch's float8_e4m3fn and
bfloat16 conversions (library routines), the numbers the P-cast pages print
(tests/golden/pcast_facts.txt), and properties of round-to-nearest-even.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_facts

FACTS = golden_facts()


def all_values():
    return oracle.e4m3_decode(np.arange(256, dtype=np.uint8))


def test_decode_matches_torch_for_all_codes():
    ours = all_values()
    ref = torch.from_numpy(np.arange(256, dtype=np.uint8)).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert nan.sum() == 2  # S.1111.111 for both signs: no infinities in E4M3FN


def test_printed_range_facts():
    v = all_values()
    finite = v[~np.isnan(v)]
    assert finite.max() == FACTS["e4m3_max_finite"]
    pos = np.sort(finite[finite > 0])
    # smallest normal: first value whose spacing to the next equals value / 8
    normals = [x for x in pos if x >= FACTS["e4m3_min_normal"]]
    assert normals[0] == FACTS["e4m3_min_normal"]
    assert pos[0] == 2.0 ** -9  # smallest subnormal, half of which is the round-to-zero threshold
    assert pos[0] / 2 == FACTS["e4m3_round_to_zero_threshold"]
    # 127 distinct non-negative finite magnitudes (0 and 126 positive values)
    assert len(set(abs(x) for x in finite.tolist())) == 127


def test_round_trip_all_finite_codes():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_decode(codes)
    ok = ~np.isnan(v)
    back = oracle.e4m3_encode(v[ok])
    assert np.array_equal(back, codes[ok])


def test_round_to_zero_threshold_and_tie():
    t = FACTS["e4m3_round_to_zero_threshold"]
    assert oracle.e4m3_encode_scalar(t) == 0            # exact tie -> even (zero)
    assert oracle.e4m3_encode_scalar(np.nextafter(np.float32(t), np.float32(1))) == 1
    assert oracle.e4m3_encode_scalar(np.nextafter(np.float32(t), np.float32(0))) == 0
    assert oracle.e4m3_encode_scalar(-t) == 0x80        # negative zero


def test_midpoints_round_to_even():
    v = all_values()
    pos = np.sort(np.unique(v[(v >= 0) & ~np.isnan(v)]))
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = (float(lo) + float(hi)) / 2.0
        c = oracle.e4m3_encode_scalar(mid)
        clo, chi = oracle.e4m3_encode_scalar(lo), oracle.e4m3_encode_scalar(hi)
        assert c == (clo if clo % 2 == 0 else chi), (lo, hi, c)
        # just off the midpoint goes to the nearer neighbour
        assert oracle.e4m3_encode_scalar(mid - (hi - lo) * 1e-3) == clo
        assert oracle.e4m3_encode_scalar(mid + (hi - lo) * 1e-3) == chi


def test_saturation_is_finite():
    for x in [448.0, 449.0, 463.99, 464.0, 480.0, 1e6, 3.4e38, math.inf]:
        assert oracle.e4m3_encode_scalar(x) == 0x7E
        assert oracle.e4m3_encode_scalar(-x) == 0xFE
    assert oracle.e4m3_encode_scalar(math.nan) & 0x7F == 0x7F


def test_encode_matches_torch_on_random_values():
    rng = np.random.default_rng(123)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(200_000) * 100).astype(np.float32),
        np.exp(rng.uniform(-16, 6, 200_000)).astype(np.float32),
    ])
    x = x[np.abs(x) < 440.0]  # below the largest finite value: torch and satfinite agree
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(300_000).astype(np.float32),
        np.exp(rng.uniform(-60, 60, 100_000)).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875], dtype=np.float32),
    ])
    ours = oracle.bf16_round_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
