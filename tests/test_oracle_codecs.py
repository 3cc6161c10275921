"""Pins of the oracle's E4M3 / E2M1 codecs against things other than itself:
the ml_dtypes library conversions (an independent RNE implementation), brute
force nearest-value search, and the format's printed extremes (max 448 for
E4M3 per the FP8 KV calibration guide, +-6 for E2M1)."""
import math

import ml_dtypes
import numpy as np
import pytest

import oracle

E4M3 = ml_dtypes.float8_e4m3fn
E2M1 = ml_dtypes.float4_e2m1fn


def all_bf16_values():
    bits = np.arange(65536, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    return x[~np.isnan(x)]


def test_e4m3_decode_matches_library_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = codes.view(E4M3).astype(np.float32)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok].view(np.uint32), ref[ok].view(np.uint32))  # signed zeros too
    assert np.flatnonzero(np.isnan(ours)).tolist() == [0x7F, 0xFF]


def test_e4m3_spot_values():
    d = oracle.e4m3_decode(np.array([0x7E, 0xFE, 0x01, 0x08, 0x38, 0x07, 0x80], np.uint8))
    assert d[0] == 448.0 and d[1] == -448.0          # max finite (the 448 of the scale formula)
    assert d[2] == 2.0 ** -9 and d[3] == 2.0 ** -6    # min subnormal, min normal
    assert d[4] == 1.0 and d[5] == 7 * 2.0 ** -9
    assert d[6] == 0.0 and math.copysign(1, d[6]) < 0


def test_e2m1_decode_matches_library_and_magnitudes():
    codes = np.arange(16, dtype=np.uint8)
    ours = oracle.e2m1_decode(codes)
    ref = codes.view(E2M1).astype(np.float32)
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    assert ours[:8].tolist() == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert (ours[8:] == -ours[:8]).all() and math.copysign(1, ours[8]) < 0


@pytest.mark.parametrize("brute", [False, True])
def test_e4m3_encode_all_bf16_inputs(brute):
    x = all_bf16_values()
    ours = oracle.e4m3_encode(x, brute_force=brute)
    sat = np.abs(x) >= 448.0
    # saturation (satfinite): every |x| >= 448, infinities included, goes to +-448
    assert np.all(ours[sat & (x > 0)] == 0x7E) and np.all(ours[sat & (x < 0)] == 0xFE)
    # elsewhere the library's round-to-nearest-even conversion
    ref = x[~sat].astype(E4M3).view(np.uint8)
    assert np.array_equal(ours[~sat], ref)


def test_e4m3_arithmetic_equals_brute_force_on_midpoints():
    vals = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2  # exact in float32 (few mantissa bits)
    x = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
                        np.nextafter(mids.astype(np.float32), np.float32(1e9)), [464.0, 460.0,
                        480.0, 3.0e38, np.inf]]).astype(np.float32)
    x = np.concatenate([x, -x])
    assert np.array_equal(oracle.e4m3_encode(x), oracle.e4m3_encode(x, brute_force=True))
    # ties go to the even mantissa: 17 is between 16 (m=0) and 18 (m=1)
    assert oracle.e4m3_encode([17.0])[0] == 0x58
    assert oracle.e4m3_encode([2.0 ** -10])[0] == 0x00  # half of the smallest subnormal
    assert oracle.e4m3_encode([3 * 2.0 ** -10])[0] == 0x02  # 1.5 steps -> 2 (even)
    assert oracle.e4m3_encode([464.0])[0] == 0x7E and oracle.e4m3_encode([-1e30])[0] == 0xFE
    assert oracle.e4m3_encode([-0.0])[0] == 0x80 and oracle.e4m3_encode([-1e-30])[0] == 0x80


@pytest.mark.parametrize("brute", [False, True])
def test_e2m1_encode_all_bf16_inputs(brute):
    x = all_bf16_values()
    ours = oracle.e2m1_encode(x, brute_force=brute)
    ref = x.astype(E2M1).view(np.uint8) & 0xF  # the library saturates to +-6 as well
    assert np.array_equal(ours, ref)


def test_e2m1_spot_values():
    x = [6.5, 100.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.1, -6.0, 5.5]
    want = [7, 7, 0, 2, 2, 4, 4, 6, 6, 8, 15, 7]
    assert oracle.e2m1_encode(x).tolist() == want
