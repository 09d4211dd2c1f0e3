"""Pins for the oracle's randomized Hadamard transform (CPU only).

Independent checks: brute-force sums with Python loops, an O(n log n) butterfly
written here, closed forms, norm preservation, the exact inverse, and exact
(correctly rounded) summation with math.fsum.
"""
import math

import numpy as np
import pytest

from hadamard_rotated_activation_b200 import workloads as wl
from oracle import paley12, rht, rht_inverse, rht_unnormalized


def _walsh_sign(i, j):
    return -1.0 if bin(i & j).count("1") % 2 else 1.0


def _entry(n, i, j):
    """Hadamard entry computed independently: Sylvester by popcount, or the
    Paley-12 x Sylvester Kronecker entry."""
    if n & (n - 1) == 0:
        return _walsh_sign(i, j)
    m = n // 12
    a, beta = divmod(i, m)
    c, delta = divmod(j, m)
    return paley12()[a, c] * _walsh_sign(beta, delta)


@pytest.mark.parametrize("n,block", [(16, 0), (24, 0), (32, 8), (48, 0)])
def test_brute_force_definition(n, block):
    """y_i = (1/sqrt(b)) sum_j H[i][j] s_j x_j per block (row-vector Y = X H^T)."""
    rng = np.random.default_rng(n)
    x = rng.standard_normal((3, n))
    s = (1 - 2 * rng.integers(0, 2, n)).astype(np.int8)
    y = rht(x, s, block)
    b = n if block == 0 else block
    for t in range(3):
        for blk in range(n // b):
            for i in range(b):
                acc = 0.0
                for j in range(b):
                    jj = blk * b + j
                    acc += _entry(b, i, j) * s[jj] * x[t, jj]
                assert y[t, blk * b + i] == pytest.approx(acc / math.sqrt(b),
                                                          rel=1e-13, abs=1e-13)


def _fwht_butterfly(v):
    """Unnormalised Sylvester transform along the last axis, in-place butterfly."""
    v = np.array(v, dtype=np.float64)
    n = v.shape[-1]
    h = 1
    while h < n:
        v = v.reshape(v.shape[:-1] + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        v = v.reshape(v.shape[:-3] + (n,))
        h *= 2
    return v


def test_dense_equals_butterfly_4096():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((8, 4096))
    s = (1 - 2 * rng.integers(0, 2, 4096)).astype(np.int8)
    want = _fwht_butterfly(x * s) / 64.0
    np.testing.assert_allclose(rht(x, s, 0), want, rtol=0, atol=1e-12)


def test_dense_equals_factored_12288():
    """H12 kron H1024 applied as a 12-point dense stage after 1024-point
    butterflies on each of the 12 segments (the slow index is the H12 one)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 12288))
    s = (1 - 2 * rng.integers(0, 2, 12288)).astype(np.int8)
    w = _fwht_butterfly((x * s).reshape(4, 12, 1024))
    h12 = paley12()
    z = np.einsum("ac,tcb->tab", h12, w).reshape(4, 12288)
    np.testing.assert_allclose(rht_unnormalized(x, s, 0), z, rtol=0, atol=1e-9)


@pytest.mark.parametrize("n,block", [(4096, 0), (4096, 128), (12288, 0), (256, 16)])
def test_norm_preserved_and_inverse(n, block):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, n)) * rng.lognormal(0, 1, n)
    s = (1 - 2 * rng.integers(0, 2, n)).astype(np.int8)
    y = rht(x, s, block)
    b = n if block == 0 else block
    nx = np.linalg.norm(x.reshape(-1, b), axis=1)
    ny = np.linalg.norm(y.reshape(-1, b), axis=1)
    np.testing.assert_allclose(ny, nx, rtol=1e-13)
    np.testing.assert_allclose(rht_inverse(y, s, block), x, rtol=0,
                               atol=1e-13 * np.max(np.abs(x)))


@pytest.mark.parametrize("n", [128, 4096, 12288])
def test_closed_forms(n):
    """x = e_0 -> y = s_0 H[:, 0] / sqrt(n) = s_0 / sqrt(n) * 1 (first column of
    Sylvester and of H12 kron H are +1 for Sylvester; for Paley the first column
    is (+1, -1, ..., -1) kron 1);  x = s (so D x = 1) -> y = H 1 / sqrt(n) =
    sqrt(n) e_0 (row sums: n for row 0, 0 otherwise)."""
    rng = np.random.default_rng(4)
    s = (1 - 2 * rng.integers(0, 2, n)).astype(np.int8)
    e0 = np.zeros((1, n))
    e0[0, 0] = 1.0
    y = rht(e0, s, 0)[0]
    if n & (n - 1) == 0:
        col = np.ones(n)
    else:
        col = np.kron(np.array([1.0] + [-1.0] * 11), np.ones(n // 12))
    np.testing.assert_allclose(y, s[0] * col / math.sqrt(n), rtol=1e-15)
    y = rht(s[None, :].astype(np.float64), s, 0)[0]
    want = np.zeros(n)
    want[0] = math.sqrt(n)
    np.testing.assert_allclose(y, want, rtol=1e-15, atol=1e-12)


def test_block_mode_is_independent_blocks():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 512))
    s = (1 - 2 * rng.integers(0, 2, 512)).astype(np.int8)
    y = rht(x, s, 128)
    for k in range(4):
        sl = slice(128 * k, 128 * (k + 1))
        np.testing.assert_array_equal(y[:, sl], rht(x[:, sl], s[sl], 0))


def test_no_signs_equals_all_plus_signs():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((2, 256))
    np.testing.assert_array_equal(rht(x, None, 128),
                                  rht(x, np.ones(256, dtype=np.int8), 128))


def test_fp64_sums_exact_on_bf16_workload_rows():
    """For bf16 inputs the oracle's float64 sums equal the correctly rounded
    exact sums (math.fsum) at the row maxima that decide the scales."""
    for key in ("c3", "c4"):
        inp = wl.make_inputs(wl.WORKLOADS[key], tokens=3)
        w = inp.workload
        s_un = rht_unnormalized(inp.values, inp.signs, w.block)
        n = w.dim
        for t in range(3):
            i = int(np.argmax(np.abs(s_un[t])))
            terms = [_entry(n, i, j) * inp.signs[j] * inp.values[t, j]
                     for j in range(n)]
            assert s_un[t, i] == math.fsum(terms)


def test_rejects_bad_block_and_signs():
    x = np.zeros((1, 96))
    with pytest.raises(ValueError):
        rht(x, None, 64)
    with pytest.raises(ValueError):
        rht(x, np.zeros(96, dtype=np.int8), 0)
