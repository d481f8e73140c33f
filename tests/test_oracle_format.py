"""Pins of the oracle's scalar formats (E2M1, E4M3, bf16) against the format
definitions, exhaustive enumeration, brute force in exact rationals and the
ml_dtypes / torch conversions.  CPU only."""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_e2m1():
    vals = {}
    with open(os.path.join(GOLDEN, "e2m1_values.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            c, v = line.split()
            vals[int(c)] = float(v)
    return vals


def _e2m1_from_bits(code):
    """E2M1 from its bit fields: sign | 2-bit exponent (bias 1) | 1-bit mantissa."""
    s, e, m = code >> 3, (code >> 1) & 3, code & 1
    mag = (m / 2.0) if e == 0 else (1 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_decode_table_all_16_codes():
    golden = _golden_e2m1()
    for code in range(16):
        v = oracle.e2m1_value(code)
        assert v == _e2m1_from_bits(code)
        assert abs(v) == golden[code & 7]
        assert math.copysign(1.0, v) == (-1.0 if code & 8 else 1.0)
        ref = float(np.array([code], dtype=np.uint8).view(ml_dtypes.float4_e2m1fn)[0])
        assert v == ref


@pytest.mark.parametrize("d", [1.0, 1.75, 0.171875, 2.0 ** -20, 3.0517578125e-05, 448 * 2.0 ** -8,
                               1.2345678])
def test_e2m1_every_value_round_trips(d):
    d = float(np.float32(d))
    for idx in range(8):
        ax = np.float32(oracle.e2m1_value(idx) * d)
        if float(ax) != oracle.e2m1_value(idx) * d:
            continue  # the product is not a float32; not a round-trip case
        assert oracle.e2m1_index_exact(float(ax), d) == idx


def _brute_e2m1_index(q: Fraction) -> int:
    """Nearest E2M1 magnitude to the rational q >= 0, ties to the even index,
    found by scanning all 8 magnitudes."""
    mags = [Fraction(v).limit_denominator(4) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    best, bestd = 0, None
    for i, m in enumerate(mags):
        dist = abs(q - m)
        if bestd is None or dist < bestd or (dist == bestd and i % 2 == 0):
            best, bestd = i, dist
    return best


def test_e2m1_exact_quotient_vs_bruteforce_sweep():
    rng = np.random.default_rng(7)
    ds = [np.float32(1.0), np.float32(1.75), np.float32(0.171875), np.float32(0.1),
          np.float32(3.7e-3)]
    for d in ds:
        # every float32 multiple k/64 * d near and at all midpoints, plus random
        qs = [Fraction(k, 64) for k in range(0, 6 * 64 + 80)]
        for q in qs:
            ax = np.float32(float(q * Fraction(float(d))))
            want = _brute_e2m1_index(Fraction(float(ax)) / Fraction(float(d)))
            assert oracle.e2m1_index_exact(float(ax), float(d)) == want, (float(ax), float(d))
        for ax in rng.uniform(0, 7 * float(d), 2000).astype(np.float32):
            want = _brute_e2m1_index(Fraction(float(ax)) / Fraction(float(d)))
            assert oracle.e2m1_index_exact(float(ax), float(d)) == want


def test_e2m1_ties_go_to_even_index():
    # the 7 midpoints with D = 1 (all exact): 0.25->0, 0.75->2, 1.25->2, 1.75->4,
    # 2.5->4, 3.5->6, 5->6; above 6 saturates to index 7
    got = [oracle.e2m1_index_exact(m, 1.0) for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 100.0)]
    assert got == [0, 2, 2, 4, 4, 6, 6, 7]


def test_e2m1_matches_ml_dtypes_rne_in_range():
    qs = np.linspace(0, 6, 6001, dtype=np.float32)
    ref = qs.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 7
    got = np.array([oracle.e2m1_index_exact(float(q), 1.0) for q in qs])
    assert np.array_equal(got, ref)


def _e4m3_from_bits(b):
    s, e, m = b >> 7, (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return math.nan
    v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
    return -v if s else v


def test_e4m3_decode_all_256_codes():
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for b in range(256):
        v = oracle.e4m3_value(b)
        if math.isnan(ref[b]):
            assert math.isnan(v) and (b & 0x7F) == 0x7F
        else:
            assert v == ref[b] == _e4m3_from_bits(b)


def test_e4m3_encode_spot_values():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(44.0) == 0x63
    assert oracle.e4m3_encode(1.0) == 0x38
    assert oracle.e4m3_encode(2.0 ** -9) == 0x01
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00  # tie with 0 -> even code 0
    assert oracle.e4m3_encode(3 * 2.0 ** -11) == 0x01  # 0.75 * 2^-9 -> nearest 2^-9
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02  # 1.5 * 2^-9: tie 1|2 -> even code 2
    assert oracle.e4m3_encode(5 * 2.0 ** -10) == 0x02  # 2.5 * 2^-9: tie 2|3 -> even code 2
    assert oracle.e4m3_encode(1000.0) == 0x7E  # saturates
    assert oracle.e4m3_encode(42.666668) == 0x63


def test_e4m3_encode_vs_ml_dtypes_sweep():
    rng = np.random.default_rng(3)
    # dense float32 sweep over [0, 448]: random + every E4M3 value and midpoint
    vals = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    sweep = np.concatenate([rng.uniform(0, 448, 20000).astype(np.float32),
                            np.exp2(rng.uniform(-12, 8.8, 20000)).astype(np.float32), vals, mids,
                            np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    sweep = sweep[(sweep >= 0) & (sweep <= 448)]
    ref = sweep.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([oracle.e4m3_encode(float(s)) for s in sweep], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(sweep[i]), int(got[i]), int(ref[i])) for i in bad[:5]]


def test_e4m3_encode_vs_bruteforce_rationals():
    finite = [Fraction(_e4m3_from_bits(b)) for b in range(127)]
    rng = np.random.default_rng(11)
    for s in np.exp2(rng.uniform(-11, 9, 3000)).astype(np.float32):
        q = Fraction(float(s))
        if q >= 448:
            want = 0x7E
        else:
            want, bestd = 0, None
            for b, v in enumerate(finite):
                d = abs(q - v)
                if bestd is None or d < bestd or (d == bestd and b % 2 == 0):
                    want, bestd = b, d
        assert oracle.e4m3_encode(float(s)) == want


def test_bf16_rne_vs_torch():
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.standard_normal(5000).astype(np.float32) * 100,
                         np.float32([1.0, -1.0, 0.0, -0.0, 3.3895314e38, 1e-40, 1.00390625,
                                     1.005859375, 1.0029296875])])
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)
