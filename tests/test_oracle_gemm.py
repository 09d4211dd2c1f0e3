"""Pins of the NVFP4 GEMM oracle and of the scale-factor layout (CPU).

* Exact brute force: rational arithmetic (fractions) of the definition on
  tiny matrices, rounded once, equals nvfp4_gemm bit for bit.
* Closed form: a one-hot row of A (value 1.0) picks one column of B.
* The pinned dequantizer: with power-of-two tensor scales every dequantized
  value is exact in fp32, so C equals the product of dequant_nvfp4 outputs.
* Computational invariance (QuaRot reviews, review 3 Questions, Y = X H^T):
  quantizing the rotated rows of X and W and multiplying gives X W^T within
  the quantization error the half-step bounds allow.
* The layout: a bijection, inverted by sf_from_mma_layout, zero padding.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import gemm


def _random_nvfp4(rng, rows, k, zero_scale=False):
    codes = rng.integers(0, 16, size=(rows, k))
    scales = rng.integers(0, 0x7F, size=(rows, k // 16)).astype(np.uint8)   # finite codes
    if zero_scale:
        scales[0, 0] = 0
        scales[-1, -1] = 1                                                  # subnormal 2^-9
    return codes, scales


def test_brute_force_exact():
    rng = np.random.default_rng(0)
    a, sa = _random_nvfp4(rng, 3, 48, zero_scale=True)
    b, sb = _random_nvfp4(rng, 2, 48, zero_scale=True)
    ta, tb = np.float32(0.0371), np.float32(3.5e-3)
    got = gemm.nvfp4_gemm(a, sa, ta, b, sb, tb)
    va = oracle.e2m1_decode(a)
    vb = oracle.e2m1_decode(b)
    fa, fb = oracle.e4m3_decode(sa), oracle.e4m3_decode(sb)
    for m in range(3):
        for n in range(2):
            acc = Fraction(0)
            for k in range(48):
                acc += (Fraction(float(va[m, k])) * Fraction(float(fa[m, k // 16])) *
                        Fraction(float(ta)) * Fraction(float(vb[n, k])) *
                        Fraction(float(fb[n, k // 16])) * Fraction(float(tb)))
            assert got[m, n] == float(acc), (m, n)


def test_one_hot_row_picks_a_column():
    rng = np.random.default_rng(1)
    b, sb = _random_nvfp4(rng, 5, 64)
    tb = np.float32(0.125)
    a = np.zeros((1, 64), dtype=np.int64)
    sa = np.zeros((1, 4), dtype=np.uint8)
    k0 = 37
    a[0, k0] = 2                      # E2M1 1.0
    sa[0, k0 // 16] = 0x38            # E4M3 1.0
    c = gemm.nvfp4_gemm(a, sa, 1.0, b, sb, tb)
    want = oracle.e2m1_decode(b[:, k0]) * oracle.e4m3_decode(sb[:, k0 // 16]) * 0.125
    assert np.array_equal(c[0], want)


def test_matches_the_dequantizer_with_exact_scales():
    rng = np.random.default_rng(2)
    a, sa = _random_nvfp4(rng, 7, 128)
    b, sb = _random_nvfp4(rng, 6, 128)
    ta, tb = np.float32(2.0 ** -7), np.float32(2.0 ** 3)
    da = oracle.dequant_nvfp4(a, sa, ta).astype(np.float64)
    db = oracle.dequant_nvfp4(b, sb, tb).astype(np.float64)
    assert np.array_equal(gemm.nvfp4_gemm(a, sa, ta, b, sb, tb), da @ db.T)
    assert np.array_equal(gemm.nvfp4_gemm_abs(a, sa, ta, b, sb, tb), np.abs(da) @ np.abs(db).T)


def test_rotation_leaves_the_product_invariant():
    rng = np.random.default_rng(3)
    n = 256
    x = rng.standard_normal((4, n)) * rng.lognormal(0, 1, n)
    w = rng.standard_normal((3, n)) / np.sqrt(n)
    s = (1 - 2 * rng.integers(0, 2, n)).astype(np.int8)
    yx, yw = oracle.rht(x, s, 0), oracle.rht(w, s, 0)
    assert np.allclose(yx @ yw.T, x @ w.T, rtol=1e-12, atol=1e-12)
    cx, bx, tx = oracle.nvfp4(yx)
    cw, bw, tw = oracle.nvfp4(yw)
    c = gemm.nvfp4_gemm(cx, bx, tx, cw, bw, tw)
    # |x_hat w_hat^T - x w^T| <= ||yx - yx_hat|| ||yw_hat|| + ||yx|| ||yw - yw_hat||, each
    # element of y - y_hat within one scale unit (half a grid gap or the saturation error)
    dx = oracle.dequant_nvfp4(cx, bx, tx).astype(np.float64)
    dw = oracle.dequant_nvfp4(cw, bw, tw).astype(np.float64)
    ux = np.repeat(oracle.e4m3_decode(bx), 16, axis=1) * np.float64(tx)
    uw = np.repeat(oracle.e4m3_decode(bw), 16, axis=1) * np.float64(tw)
    ex = np.sqrt((np.maximum(ux, 6 * np.float64(tx) * 2.0 ** -10) ** 2).sum(1))
    ew = np.sqrt((np.maximum(uw, 6 * np.float64(tw) * 2.0 ** -10) ** 2).sum(1))
    bound = (ex[:, None] * np.linalg.norm(dw, axis=1)[None, :] +
             np.linalg.norm(yx, axis=1)[:, None] * ew[None, :])
    assert np.all(np.abs(c - x @ w.T) <= bound * 1.0001)
    assert np.abs(c - x @ w.T).max() < 0.5 * np.abs(x @ w.T).max()   # not vacuous


@pytest.mark.parametrize("rows,kc", [(128, 4), (130, 5), (1, 1), (300, 256), (256, 12)])
def test_sf_layout_is_a_padded_bijection(rows, kc):
    rng = np.random.default_rng(rows * 1000 + kc)
    s = rng.integers(1, 0x7F, size=(rows, kc)).astype(np.uint8)
    flat = gemm.sf_mma_layout(s)
    pr, pk = -(-rows // 128) * 128, -(-kc // 4) * 4
    assert flat.shape == (pr * pk,)
    assert np.array_equal(gemm.sf_from_mma_layout(flat, rows, kc), s)
    # every real scale appears once; everything else is zero padding
    assert np.count_nonzero(flat) == rows * kc
    ids = np.arange(rows * kc).reshape(rows, kc)
    perm = gemm.sf_mma_layout((ids % 251 + 1).astype(np.uint8))
    assert sorted(perm[perm > 0].tolist()) == sorted((ids.reshape(-1) % 251 + 1).tolist())


def test_sf_layout_atoms():
    """Inside one 512-byte atom a row's four scales are contiguous; rows r and
    r + 32 are 4 bytes apart, rows r and r + 1 are 16 bytes apart; the next
    four 16-blocks start the next atom."""
    rows, kc = 128, 8
    s = np.zeros((rows, kc), dtype=np.uint8)
    s[0, 0:4] = [1, 2, 3, 4]
    s[1, 0] = 5
    s[32, 0] = 6
    s[0, 4] = 7
    flat = gemm.sf_mma_layout(s)
    assert flat[0:4].tolist() == [1, 2, 3, 4]
    assert flat[16] == 5 and flat[4] == 6 and flat[512] == 7
