"""Pins for the oracle's quantizers (CPU only): hand-worked examples from the
format definitions, half-step error bounds, invariants, storage accounting and
special cases."""
import numpy as np
import pytest

from oracle import (
    dequant_int4_asym, dequant_int4_sym, dequant_mxfp4, dequant_nvfp4, e2m1_decode,
    e4m3_decode, int4_asym_group, int4_sym_per_token, mxfp4, mxfp4_exponents, nvfp4,
    pack_nibbles, rht, unpack_nibbles,
)
from oracle.quant import int4_from_nibble
from hadamard_rotated_activation_b200 import workloads as wl


def _section(rows, k):
    return rows[k]


def test_int4_sym_hand_example(golden):
    rows = golden("int4_sym_example.txt")
    y = np.array([[float(v) for v in rows[0]]])
    q, s = int4_sym_per_token(y)
    assert s.view(np.uint32)[0] == int(rows[1][0], 16)
    assert list(q[0]) == [int(v) for v in rows[2]]
    assert list(pack_nibbles(q)[0]) == [int(v, 16) for v in rows[3]]


def test_nvfp4_hand_example(golden):
    rows = golden("nvfp4_example.txt")
    y = np.array([[float(v) for v in rows[0]]])
    codes, sb, t = nvfp4(y, tensor_scale=float(rows[1][0]))
    assert sb[0, 0] == int(rows[2][0], 16)
    assert list(codes[0]) == [int(v, 16) for v in rows[3]]
    assert list(pack_nibbles(codes)[0]) == [int(v, 16) for v in rows[4]]


def test_int4_asym_hand_example(golden):
    rows = golden("int4_asym_example.txt")
    y = np.array([[float(v) for v in rows[0]]])
    g = int(rows[1][0])
    u, s16, z16 = int4_asym_group(y, g)
    assert s16.view(np.uint16)[0, 0] == int(rows[2][0], 16)
    assert z16.view(np.uint16)[0, 0] == int(rows[2][1], 16)
    assert list(u[0]) == [int(v) for v in rows[3]]


def test_nvfp4_dynamic_tensor_scale_closed_form():
    y = np.zeros((2, 32))
    y[1, 5] = -2688.0
    _, _, t = nvfp4(y)
    assert t == np.float32(1.0)


def test_storage_bits(golden):
    want = {k: float(v) for k, v in golden("storage.txt")}
    t, n = 4, 4096
    y = np.random.default_rng(0).standard_normal((t, n))
    codes, sb, _ = nvfp4(y)
    bits = (pack_nibbles(codes).nbytes + sb.nbytes) * 8 / (t * n)
    assert bits == want["nvfp4"]
    q, s = int4_sym_per_token(y)
    assert (pack_nibbles(q).nbytes + s.nbytes) * 8 / (t * n) == want["int4_sym_4096"]
    u, s16, z16 = int4_asym_group(y, 128)
    assert (pack_nibbles(u).nbytes + s16.nbytes + z16.nbytes) * 8 / (t * n) == \
        want["int4_asym_g128"]


def test_pack_unpack_roundtrip():
    rng = np.random.default_rng(1)
    c = rng.integers(0, 16, (5, 64))
    assert np.array_equal(unpack_nibbles(pack_nibbles(c)), c)
    q = rng.integers(-8, 8, (5, 64))
    assert np.array_equal(int4_from_nibble(unpack_nibbles(pack_nibbles(q))), q)


def _rotated(key, tokens):
    inp = wl.make_inputs(wl.WORKLOADS[key], tokens=tokens)
    w = inp.workload
    return rht(inp.values, inp.signs, w.block)


@pytest.mark.parametrize("key", ["c1", "c3"])
def test_int4_sym_half_step_bound(key):
    y = _rotated(key, 16)
    q, s = int4_sym_per_token(y)
    assert q.min() >= -7 and q.max() <= 7          # -8 never produced
    deq = dequant_int4_sym(q, s).astype(np.float64)
    s64 = s.astype(np.float64)[:, None]
    # half a step, plus the fp32 rounding of the dequantized value
    assert np.all(np.abs(y - deq) <= s64 / 2 + np.abs(deq) * 2.0 ** -24 + 1e-300)
    # amax element maps to +-7 exactly
    am = np.argmax(np.abs(y), axis=1)
    assert np.all(np.abs(q[np.arange(len(q)), am]) == 7)


def test_int4_sym_zero_row_and_ties():
    y = np.zeros((2, 8))
    y[1] = [7, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5]   # scale 1: exact ties
    q, s = int4_sym_per_token(y)
    assert s[0] == 0 and np.all(q[0] == 0)
    assert list(q[1]) == [7, 0, 2, 2, 0, -2, -2, 4]


@pytest.mark.parametrize("key", ["c2", "c4"])
def test_nvfp4_half_step_bound(key):
    y = _rotated(key, 16)
    codes, sb, t = nvfp4(y)
    deq = dequant_nvfp4(codes, sb, t).astype(np.float64)
    sbv = e4m3_decode(sb)
    step = np.repeat(sbv, 16, axis=1) * np.float64(t)           # value of 1 unit
    v = np.abs(y) / np.where(step > 0, step, 1)
    # local half gap of the E2M1 grid at the decoded value
    mag = np.abs(e2m1_decode(codes))
    half_gap = np.where(mag < 2, 0.25, np.where(mag < 4, 0.5, 1.0))
    err = np.abs(y - deq)
    normal = np.repeat(sbv >= 2.0 ** -6, 16, axis=1)
    unsat = v <= 6.0
    ok = err <= half_gap * step + np.abs(deq) * 2.0 ** -24
    assert np.all(ok[normal & unsat])
    # saturation: r rounds to E4M3 at most 1/16 relative downwards, so
    # |v| <= 6 / (1 - 2^-4) and the error stays below one E2M1 top half-gap
    sat = normal & ~unsat
    assert np.all(v[sat] <= 6.0 / (1 - 2.0 ** -4) + 1e-12)
    assert np.all(err[sat] <= 1.0 * step[sat])
    # the block maximum is within the top of the grid
    assert np.all(np.max(mag.reshape(len(y), -1, 16), axis=2)[sbv > 0] >= 4.0)


def test_nvfp4_zero_block_and_sign_of_zero():
    y = np.zeros((1, 32))
    y[0, 16:] = np.linspace(-1, 1, 16)
    y[0, 17] = -1e-6                               # tiny negative -> 0x8
    codes, sb, t = nvfp4(y)
    assert sb[0, 0] == 0 and np.all(codes[0, :16] == 0)
    assert codes[0, 17] == 0x8


@pytest.mark.parametrize("key", ["c5"])
def test_int4_asym_half_step_bound(key):
    y = _rotated(key, 16)
    u, s16, z16 = int4_asym_group(y, 128)
    assert u.min() >= 0 and u.max() <= 15
    deq = dequant_int4_asym(u, s16, z16, 128).astype(np.float64)
    s = np.repeat(s16.astype(np.float64), 128, axis=1)
    z = np.repeat(z16.astype(np.float64), 128, axis=1)
    raw = np.rint(y / s) + z
    unclamped = (raw >= 0) & (raw <= 15)
    err = np.abs(y - deq)
    assert np.all(err[unclamped] <= s[unclamped] / 2 + np.abs(deq[unclamped]) * 2.0 ** -24)
    # z is an exact small integer
    assert np.all(z16.astype(np.float64) == np.rint(z16.astype(np.float64)))
    assert unclamped.mean() > 0.999


def test_int4_asym_constant_group():
    y = np.full((1, 256), 3.0)
    y[0, 128:] = np.linspace(-2, 5, 128)
    u, s16, z16 = int4_asym_group(y, 128)
    assert s16[0, 0] == 0 and z16[0, 0] == 0 and np.all(u[0, :128] == 0)
    assert u[0, 128] == 0 and u[0, 255] == 15


# ------------------------------------------------------------------ MXFP4
def test_mxfp4_hand_example():
    """Worked by hand from the MX definition: X = 2^(floor(log2 amax) - 2)."""
    y = np.zeros((2, 64))
    y[0, 32] = 1.0
    y[0, 33:64] = 0.5          # amax 1: e = -2, X = 1/4, v = 4 and 2
    y[1, 0] = -6.0             # amax 6: e = 0, X = 1, v = -6
    y[1, 1] = 0.75             # v = 0.75: tie between 0.5 and 1, even index -> 1
    y[1, 32:64] = 3.9          # amax 3.9: e = -1, X = 1/2, v = 7.8 saturates to 6
    codes, sc = mxfp4(y)
    assert sc.tolist() == [[0, 125], [127, 126]]
    assert np.all(codes[0, :32] == 0)                    # all-zero block
    assert codes[0, 32] == 6 and np.all(codes[0, 33:64] == 4)
    assert codes[1, 0] == 15 and codes[1, 1] == 2
    assert np.all(codes[1, 32:] == 7)
    deq = dequant_mxfp4(codes, sc)
    assert deq[1, 0] == -6.0 and deq[1, 1] == 1.0 and deq[1, 32] == 3.0


def test_mxfp4_exponent_brackets_block_max():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((6, 256)) * np.exp(rng.uniform(-40, 40, (6, 1)))
    y[0, :32] = 2.0 ** 7                   # amax exactly a power of two
    y[1, :32] = -np.nextafter(2.0 ** 7, 0)  # just below one
    e = mxfp4_exponents(y)
    amax = np.max(np.abs(y.reshape(6, 8, 32)), axis=2)
    lo, hi = np.ldexp(1.0, e + 2), np.ldexp(1.0, e + 3)
    assert np.all((lo <= amax) & (amax < hi))
    assert e[0, 0] == 5 and e[1, 0] == 4


def test_mxfp4_half_step_bound_and_saturation():
    y = _rotated("c4", 16)
    codes, sc = mxfp4(y)
    deq = dequant_mxfp4(codes, sc).astype(np.float64)
    X = np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1)
    v = np.abs(y) / X
    mag = np.abs(e2m1_decode(codes))
    half_gap = np.where(mag < 2, 0.25, np.where(mag < 4, 0.5, 1.0))
    err = np.abs(y - deq)
    unsat = v <= 6.0
    assert np.all(err[unsat] <= half_gap[unsat] * X[unsat])
    # v < 8 always (amax < 2^(e+3)); saturated values lose less than 2 X
    assert np.all(v < 8.0)
    assert np.all(err[~unsat] < 2.0 * X[~unsat])
    assert np.all(mag[~unsat] == 6.0)


def test_mxfp4_power_of_two_scaling_and_clamps():
    rng = np.random.default_rng(6)
    y = rng.standard_normal((3, 64))
    c0, s0 = mxfp4(y)
    c1, s1 = mxfp4(y * 2.0 ** 9)
    assert np.array_equal(c0, c1) and np.all(s1.astype(int) - s0.astype(int) == 9)
    tiny = np.full((1, 32), 2.0 ** -140)
    c, s = mxfp4(tiny)
    assert s[0, 0] == 0                  # e clamped to -127
    huge = np.full((1, 32), 2.0 ** 200)
    c, s = mxfp4(huge)
    assert s[0, 0] == 254 and np.all(c == 7)   # e clamped to 127, v saturates
    neg = np.zeros((1, 32))
    neg[0, 0] = 1.0
    neg[0, 1] = -1e-9                  # rounds to zero: sign bit kept (0x8)
    c, s = mxfp4(neg)
    assert c[0, 1] == 0x8 and c[0, 2] == 0
