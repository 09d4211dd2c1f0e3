"""The comparison helpers themselves, on the CPU: the oracle's own result
passes with zero counts; a code flipped far from any rounding boundary, or a
wrong scale, fails; a code flipped where the pre-rounding value sits on a
boundary is counted as near, not failed.  (The parity contract: scales bit
for bit, codes bit for bit except within 1e-5 relative of a boundary, such
cases counted and reported.)"""
import numpy as np
import pytest

import oracle
from oracle.quant import int4_from_nibble
import parity as P


def _rows(n=4, dim=256, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, dim)) * rng.lognormal(0, 1, dim)
    s = (1 - 2 * rng.integers(0, 2, dim)).astype(np.int8)
    return oracle.rht(x, s, 0)


def test_int4_sym_counts():
    y = _rows()
    q, sc = oracle.int4_sym_per_token(y)
    codes = oracle.pack_nibbles(q)
    c = P.check_int4_sym(codes, sc, y, name=False)
    assert (c.rows, c.codes, c.scales, c.scale_mismatch, c.near, c.bad) == (4, 1024, 4, 0, 0, 0)
    # a far flip: value well inside a rounding cell
    v = y / sc.astype(np.float64)[:, None]
    i, j = np.unravel_index(np.argmin(np.abs(v - np.rint(v))), v.shape)
    q2 = q.copy()
    q2[i, j] = q2[i, j] + 1 if q2[i, j] < 7 else q2[i, j] - 1
    with pytest.raises(AssertionError):
        P.check_int4_sym(oracle.pack_nibbles(q2), sc, y, name=False)
    assert P.check_int4_sym(oracle.pack_nibbles(q2), sc, y, strict=False, name=False).bad == 1
    # a wrong scale
    sc2 = sc.copy()
    sc2[1] = np.nextafter(sc2[1], np.float32(np.inf))
    with pytest.raises(AssertionError):
        P.check_int4_sym(codes, sc2, y, name=False)


def test_int4_sym_near_boundary_is_counted():
    # one value exactly on a half-integer in code units: either neighbour is accepted
    y = _rows(1)
    q, sc = oracle.int4_sym_per_token(y)
    j = int(np.argmin(np.abs(y[0])))
    y[0, j] = 2.5 * np.float64(sc[0])                   # rint -> 2 (ties to even)
    q, sc2 = oracle.int4_sym_per_token(y)
    assert sc2[0] == sc[0] and q[0, j] == 2
    q_alt = q.copy()
    q_alt[0, j] = 3
    c = P.check_int4_sym(oracle.pack_nibbles(q_alt), sc, y, name=False)
    assert (c.near, c.bad) == (1, 0)


def test_nvfp4_counts_and_near():
    y = _rows(3, 512, 1)
    codes, bs, t = oracle.nvfp4(y)
    packed = oracle.pack_nibbles(codes)
    c = P.check_nvfp4(packed, bs, t, y, name=False)
    assert (c.rows, c.codes, c.scales, c.scale_mismatch, c.near, c.bad) == \
        (3, 1536, 3 * 32 + 1, 0, 0, 0)
    # place one value on the 2.5 midpoint of its block's grid: 2 and 3 both pass
    den = oracle.e4m3_decode(bs).astype(np.float64) * np.float64(t)
    r, b = 0, 5
    k = b * 16 + int(np.argmin(np.abs(y[r, b * 16:(b + 1) * 16])))
    y2 = y.copy()
    y2[r, k] = 2.5 * den[r, b]
    c2, bs2, t2 = oracle.nvfp4(y2, t)
    assert np.array_equal(bs2, bs)
    alt = c2.copy()
    alt[r, k] = 5 if c2[r, k] == 4 else 4               # E2M1 index 4 = 2.0, 5 = 3.0
    cnt = P.check_nvfp4(oracle.pack_nibbles(alt), bs, t, y2, tensor_scale=t, name=False)
    assert (cnt.near, cnt.bad) == (1, 0)
    # a far flip fails
    far = c2.copy()
    far[2, 0] ^= 0x4
    with pytest.raises(AssertionError):
        P.check_nvfp4(oracle.pack_nibbles(far), bs, t, y2, tensor_scale=t, name=False)


def test_asym_and_mxfp4_counts():
    y = _rows(2, 256, 2)
    u, s16, z16 = oracle.int4_asym_group(y, 128)
    c = P.check_int4_asym(oracle.pack_nibbles(u), s16, z16, y, 128, name=False)
    assert (c.rows, c.codes, c.scales, c.scale_mismatch, c.bad) == (2, 512, 8, 0, 0)
    z2 = z16.copy()
    z2[0, 0] = z2[0, 0] + np.float16(1)
    with pytest.raises(AssertionError):
        P.check_int4_asym(oracle.pack_nibbles(u), s16, z2, y, 128, name=False)
    mc, ms = oracle.mxfp4(y)
    c = P.check_mxfp4(oracle.pack_nibbles(mc), ms, y, name=False)
    assert (c.rows, c.codes, c.scales, c.bad) == (2, 512, 16, 0)


def test_record_and_chunks():
    P.REPORT.pop("unit", None)
    P.record("unit", P.Counts(rows=2, codes=8))
    P.record("unit", P.Counts(rows=1, codes=4, near=1))
    assert P.REPORT.pop("unit") == P.Counts(rows=3, codes=12, near=1)
    spans = list(P.row_chunks(10, 4, budget=12))
    assert spans == [(0, 3), (3, 6), (6, 9), (9, 10)]
    q = int4_from_nibble(np.array([0, 7, 8, 15]))
    assert q.tolist() == [0, 7, -8, -1]
