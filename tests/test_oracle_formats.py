"""Pins of the oracle's software number formats.

Hand-worked encodings follow the format definitions (OCP FP8 E4M3FN; FP4
E2M1; bf16) used for the NVFP4 / FP8 tiers of "Triage" (zhuanzhiai paper page,
abstract).  Each expected code below is derived in its comment.  Independent
cross-checks use ml_dtypes and torch conversions on in-range values.
"""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F


# (value, code, derivation)
E4M3_HAND = [
    (1.0, 0x38, "exp 0 -> field 7 = 0b0111, mant 0: 0.0111.000"),
    (448.0, 0x7E, "1.75*2^8: field 15, mant 6: 0.1111.110"),
    (-2.0, 0xC0, "sign 1, exp 1 -> field 8: 1.1000.000"),
    (2.0 ** -6, 0x08, "smallest normal: field 1, mant 0"),
    (2.0 ** -9, 0x01, "smallest subnormal: 1 * 2^-9"),
    (2.0 ** -10, 0x00, "half of 2^-9: tie, goes to even 0"),
    (3 * 2.0 ** -10, 0x02, "1.5 * 2^-9: tie between 1 and 2, even is 2"),
    (1.0625, 0x38, "1 + 1/16 is halfway 1.0 / 1.125: even mantissa 0"),
    (1.1875, 0x3A, "halfway 1.125 / 1.25: even mantissa 2 -> 1.25"),
    (0.3, 0x2A, "0.3 = 1.2*2^-2, nearest 1.25*2^-2 = 0.3125: field 5 mant 2"),
    (1.6667, 0x3D, "nearest 1.625: mant 5"),
    (470.0, 0x7E, "above 448: satfinite clamps to 448"),
    (-1e-5, 0x80, "rounds to zero, keeps its sign"),
]


@pytest.mark.parametrize("x,code,why", E4M3_HAND)
def test_e4m3_hand_worked(x, code, why):
    assert int(F.e4m3_encode(np.array([x]))[0]) == code, why


def test_e4m3_all_codes_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert len(codes) == 254
    vals = F.e4m3_decode(codes)
    assert np.all(np.isfinite(vals))
    np.testing.assert_array_equal(F.e4m3_encode(vals), codes)


def test_e4m3_midpoints_go_to_even():
    pos = np.arange(0, 0x7F, dtype=np.uint8)          # 0 .. 0x7E, increasing values
    v = F.e4m3_decode(pos)
    mid = 0.5 * (v[:-1] + v[1:])
    got = F.e4m3_encode(mid)
    lo, hi = pos[:-1], pos[1:]
    want = np.where(lo % 2 == 0, lo, hi)
    np.testing.assert_array_equal(got, want)


def test_e4m3_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.uniform(-4, 2, 20000),
                        rng.uniform(-448, 448, 5000)])
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(F.e4m3_encode(x), ref)
    np.testing.assert_array_equal(F.e4m3_round(x), x.astype(ml_dtypes.float8_e4m3fn).astype(np.float64))


E2M1_HAND = [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
    (7.0, 6.0), (0.4, 0.5), (-1.2, -1.0), (100.0, 6.0), (5.5, 6.0),
]


@pytest.mark.parametrize("x,want", E2M1_HAND)
def test_e2m1_hand_worked(x, want):
    # grid {0, .5, 1, 1.5, 2, 3, 4, 6}; ties to the even code (mantissa bit 0)
    assert float(F.e2m1_round(np.array([x]))[0]) == want


def test_e2m1_codes():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    np.testing.assert_array_equal(F.e2m1_encode(np.array(grid)), np.arange(8))
    np.testing.assert_array_equal(F.e2m1_encode(-np.array(grid[1:])), np.arange(1, 8) | 8)
    assert int(F.e2m1_encode(np.array([-1.2]))[0]) == 0xA
    codes = np.arange(16, dtype=np.uint8)
    vals = F.e2m1_decode(codes)
    back = F.e2m1_encode(vals)
    np.testing.assert_array_equal(back, codes)


def test_e2m1_midpoints_go_to_even():
    v = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mid = 0.5 * (v[:-1] + v[1:])
    got = F.e2m1_encode(mid)
    lo, hi = np.arange(7), np.arange(1, 8)
    np.testing.assert_array_equal(got, np.where(lo % 2 == 0, lo, hi))


def test_e2m1_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(2)
    x = rng.uniform(-6, 6, 20000)
    ref = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(F.e2m1_round(x), ref)


def test_bf16_matches_torch():
    rng = np.random.default_rng(3)
    x = (rng.normal(size=50000) * 10.0 ** rng.uniform(-30, 30, 50000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(F.bf16_rne(x.astype(np.float64)), ref)


def test_bf16_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even mantissa (1.0) wins;
    # 1 + 3*2^-8 lies halfway between 1+2^-7 and 1+2^-6: 1+2^-6 (even) wins.
    assert F.bf16_rne(np.array([1 + 2 ** -8]))[0] == 1.0
    assert F.bf16_rne(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def test_ue4m3():
    assert int(F.ue4m3_encode(np.array([1.0]))[0]) == 0x38
    assert float(F.ue4m3_decode(np.array([0x3D]))[0]) == 1.625
    with pytest.raises(ValueError):
        F.ue4m3_encode(np.array([-1.0]))
