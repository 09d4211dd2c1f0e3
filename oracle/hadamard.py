"""Hadamard matrices for the oracle (test infrastructure only).

Sources:
  * QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs (reviews), review 1
    Summary: the online Hadamard is run with the Walsh-Hadamard algorithm.  The
    Walsh-Hadamard (Sylvester) matrix in natural order is
    H[i][j] = (-1)^popcount(i & j), the matrix an in-place fast transform
    produces without any reordering.
  * Bug: Qwen3-8B integration issue (KronQ #2), Model Details table:
    intermediate_size 12288 = 12 x 1024 is "Hadamard-compatible", i.e. a
    Kronecker product of an order-12 Hadamard and an order-1024 one.  The pages
    do not say which order-12 matrix.  Reading: Paley construction I with
    q = 11, H12 as the outer (slow-index) factor, in the order the phrase
    "12 x 1024" names the factors.

The matrices are built from their formulas every time; no table is stored.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np


def _is_pow2(n: int) -> bool:
    return n >= 1 and (n & (n - 1)) == 0


def sylvester(n: int) -> np.ndarray:
    """Sylvester-Hadamard matrix of order n = 2^k in natural order (float64).

    H[i][j] = (-1)^popcount(i & j).  Symmetric, H . H^T = n I.
    """
    if not _is_pow2(n):
        raise ValueError(f"Sylvester order must be a power of two, got {n}")
    idx = np.arange(n, dtype=np.int64)
    a = idx[:, None] & idx[None, :]
    parity = np.zeros_like(a)
    while np.any(a):
        parity ^= a & 1
        a >>= 1
    return np.where(parity == 0, 1.0, -1.0)


def quadratic_residues(q: int) -> frozenset:
    """Non-zero quadratic residues modulo a prime q."""
    return frozenset((k * k) % q for k in range(1, q))


def paley12() -> np.ndarray:
    """Order-12 Hadamard matrix by Paley construction I with q = 11.

    chi(0) = 0, chi(a) = +1 if a is a non-zero square mod 11, else -1.
    Jacobsthal matrix Q[i][j] = chi(j - i) for i, j in 0..10.
    S = [[0, 1^T], [-1, Q]] (skew-symmetric because q = 3 mod 4),
    H12 = I + S.  Then H12 . H12^T = 12 I; H12 is not symmetric; its first row
    is all +1 and every other row sums to 0.
    """
    q = 11
    res = quadratic_residues(q)

    def chi(a: int) -> int:
        a %= q
        if a == 0:
            return 0
        return 1 if a in res else -1

    s = np.zeros((q + 1, q + 1))
    s[0, 1:] = 1.0
    s[1:, 0] = -1.0
    for i in range(q):
        for j in range(q):
            s[1 + i, 1 + j] = chi(j - i)
    return np.eye(q + 1) + s


@lru_cache(maxsize=8)
def _hadamard_cached(n: int) -> np.ndarray:
    if _is_pow2(n):
        h = sylvester(n)
    elif n % 12 == 0 and _is_pow2(n // 12):
        h = np.kron(paley12(), sylvester(n // 12))
    else:
        raise ValueError(f"no Hadamard construction for order {n} "
                         "(supported: 2^k and 12 * 2^k)")
    h.setflags(write=False)
    return h


def hadamard(n: int) -> np.ndarray:
    """Dense Hadamard matrix of order n (read-only float64 array).

    n = 2^k: Sylvester.  n = 12 * 2^k: kron(Paley-12, Sylvester(2^k)), i.e.
    K[a*2^k + beta][c*2^k + delta] = H12[a][c] * H[beta][delta].
    """
    return _hadamard_cached(int(n))
