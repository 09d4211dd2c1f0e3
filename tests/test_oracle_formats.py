"""Pins for the oracle's number formats (CPU only): exhaustive tables, the
format specifications' anchor values, tie cases, and a brute-force nearest
search for fp16."""
import math

import numpy as np
import pytest

from oracle import E2M1_GRID, e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, fp16_round


def test_e2m1_table_matches_spec(golden):
    for code, val in golden("e2m1_table.txt"):
        got = e2m1_decode(np.array([int(code)]))[0]
        assert got == float(val)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(val))


def test_e2m1_roundtrip_all_codes():
    # every code except 0x8 (-0) round-trips; the sign bit is set only for
    # values below zero, so -0.0 encodes as 0x0
    codes = np.array([c for c in range(16) if c != 8])
    assert np.array_equal(e2m1_encode(e2m1_decode(codes)), codes)
    assert e2m1_encode(np.array([-0.0]))[0] == 0x0


@pytest.mark.parametrize("v,code", [
    (0.25, 0x0), (0.2500001, 0x1), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4),
    (2.5, 0x4), (3.5, 0x6), (5.0, 0x6), (5.0000001, 0x7), (6.0, 0x7), (7.0, 0x7),
    (1e9, 0x7), (-0.1, 0x8), (-0.25, 0x8), (-5.0, 0xE), (-100.0, 0xF), (0.0, 0x0),
])
def test_e2m1_rne_ties_and_saturation(v, code):
    assert e2m1_encode(np.array([v]))[0] == code


def test_e2m1_nearest_against_brute_force():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-8, 8, 20000), np.arange(-8, 8.25, 0.25)])
    got = e2m1_decode(e2m1_encode(v))
    for x, g in zip(v, got):
        best = min(abs(abs(x) - q) for q in E2M1_GRID)
        assert abs(abs(x) - abs(g)) == best or abs(x) > 6


def test_e4m3_anchors(golden):
    for hexcode, val in golden("e4m3_anchors.txt"):
        got = e4m3_decode(np.array([int(hexcode, 16)]))[0]
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val)
            assert math.copysign(1.0, got) == math.copysign(1.0, float(val))


def test_e4m3_monotone_and_roundtrip():
    v = e4m3_decode(np.arange(127))
    assert np.all(np.diff(v) > 0)
    assert np.array_equal(e4m3_encode(v), np.arange(127))
    # negative codes mirror positive ones
    assert np.array_equal(e4m3_decode(np.arange(128, 255)), -v)


@pytest.mark.parametrize("r,code", [
    (1.0625, 0x38),          # midpoint of 1.0 (0x38) and 1.125 (0x39): even
    (1.1875, 0x3A),          # midpoint of 1.125 and 1.25: even 0x3A
    (2.0 ** -10, 0x00),      # midpoint of 0 and 2^-9: even 0
    (1.5 * 2.0 ** -10, 0x01),
    (3 * 2.0 ** -10, 0x02),  # midpoint of 2^-9 and 2*2^-9: even 0x02
    (448.0, 0x7E), (460.0, 0x7E), (1e6, 0x7E), (0.0, 0x00),
])
def test_e4m3_rne_ties_and_saturation(r, code):
    assert e4m3_encode(np.array([r]))[0] == code


def test_e4m3_nearest_against_brute_force():
    rng = np.random.default_rng(1)
    r = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(500.0), 20000))
    enc = e4m3_encode(r)
    table = e4m3_decode(np.arange(127))
    for x, c in zip(r, enc):
        d = np.abs(table - min(x, 448.0))
        assert d[c] == d.min()


def _all_finite_fp16():
    bits = np.arange(0, 0x7C00, dtype=np.uint16)   # +0 .. max finite
    return bits.view(np.float16).astype(np.float64)


def test_fp16_round_against_brute_force():
    table = _all_finite_fp16()
    rng = np.random.default_rng(2)
    v = np.concatenate([
        np.exp(rng.uniform(np.log(1e-7), np.log(6e4), 5000)),
        (table[1:2000] + table[0:1999]) / 2,          # exact midpoints
    ])
    got = fp16_round(v).astype(np.float64)
    for x, g in zip(v, got):
        i = np.searchsorted(table, x)
        lo, hi = table[max(i - 1, 0)], table[min(i, len(table) - 1)]
        if x - lo < hi - x:
            want = lo
        elif hi - x < x - lo:
            want = hi
        else:   # tie: even mantissa
            lo_bits = np.float16(lo).view(np.uint16)
            want = lo if lo_bits % 2 == 0 else hi
        assert g == want, (x, g, want)
