"""Pins for the oracle's Hadamard matrices (CPU only).

Each check uses a construction or fact independent of the oracle's code:
the recursive Sylvester doubling, brute-force squares mod 11, Python-integer
popcounts, orthogonality.
"""
import numpy as np
import pytest

from oracle import hadamard, paley12, quadratic_residues, sylvester


def _sylvester_recursive(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256, 1024])
def test_sylvester_equals_recursive_doubling(n):
    assert np.array_equal(sylvester(n), _sylvester_recursive(n))


@pytest.mark.parametrize("n", [2, 16, 128, 4096])
def test_sylvester_orthogonal_symmetric(n):
    h = sylvester(n)
    assert np.array_equal(h @ h.T, n * np.eye(n))
    assert np.array_equal(h, h.T)
    assert np.all(h[0] == 1) and np.all(h[:, 0] == 1)


def test_sylvester_natural_order_rows():
    h = sylvester(8)
    # row 1 alternates (bit 0 of j), row 2 pairs, row 4 halves
    assert list(h[1]) == [1, -1, 1, -1, 1, -1, 1, -1]
    assert list(h[2]) == [1, 1, -1, -1, 1, 1, -1, -1]
    assert list(h[4]) == [1, 1, 1, 1, -1, -1, -1, -1]


def test_quadratic_residues_mod_11():
    brute = {x for x in range(1, 11) if any((k * k - x) % 11 == 0 for k in range(11))}
    assert quadratic_residues(11) == frozenset(brute) == frozenset({1, 3, 4, 5, 9})


def test_paley12_properties():
    h = paley12()
    assert h.shape == (12, 12)
    assert set(np.unique(h)) == {-1.0, 1.0}
    assert np.array_equal(h @ h.T, 12 * np.eye(12))
    assert np.array_equal(h.T @ h, 12 * np.eye(12))
    assert not np.array_equal(h, h.T)            # not symmetric
    s = h - np.eye(12)
    assert np.array_equal(s, -s.T)                # I + skew-symmetric
    assert np.all(h[0] == 1)                      # first row all +1
    assert np.all(h[1:].sum(axis=1) == 0)         # other rows sum to 0
    # Jacobsthal core is circulant: Q[i][j] depends on j - i mod 11 only
    q = h[1:, 1:] - np.eye(11)
    for i in range(11):
        assert np.array_equal(np.roll(q[0], i), q[i])


def test_kronecker_small_matches_entrywise_formula():
    h12, h4 = paley12(), sylvester(4)
    k = hadamard(48)
    for a in range(12):
        for beta in range(4):
            for c in range(12):
                for delta in range(4):
                    want = h12[a, c] * (-1) ** bin(beta & delta).count("1")
                    assert k[a * 4 + beta, c * 4 + delta] == want


def test_kronecker_768_orthogonal():
    k = hadamard(12 * 64)
    assert np.array_equal(k @ k.T, 768 * np.eye(768))


def test_kronecker_12288_sampled_entries_and_rows():
    """H12 kron H1024 (the 12 x 1024 'Hadamard-compatible' size): sampled
    entries against the entrywise formula with Python-int popcounts, and
    sampled row pairs orthogonal."""
    k = hadamard(12288)
    h12 = paley12()
    rng = np.random.default_rng(0)
    for _ in range(2000):
        i, j = rng.integers(0, 12288, size=2)
        a, beta = divmod(int(i), 1024)
        c, delta = divmod(int(j), 1024)
        want = h12[a, c] * (-1) ** bin(beta & delta).count("1")
        assert k[i, j] == want
    rows = rng.integers(0, 12288, size=(64, 2))
    for i, j in rows:
        d = float(k[i] @ k[j])
        assert d == (12288.0 if i == j else 0.0)


def test_unsupported_orders_raise():
    for n in (3, 6, 20, 24 * 3, 172):
        with pytest.raises(ValueError):
            hadamard(n)
