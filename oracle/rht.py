"""Randomized Hadamard transform (RHT) of activation rows, fp64 dense (oracle).

Test infrastructure only.

Sources:
  * QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs (reviews), review 2
    Summary: the randomized Hadamard transform, fully invertible up to machine
    epsilon, applied to activations to spread outliers.
  * Same page, review 3 Questions: the Hadamard block computes Y = X H^T
    (row-vector convention).  With the random +-1 diagonal D this reads
    y_row = x_row . D . H^T, i.e. y_i = sum_j H[i][j] s_j x_j.
  * Methodology checks for NVFP4 W4A4 on Qwen3-8B (forum thread),
    discrete_descent's note on block-Hadamard-128: an independent H_128 on each
    128-column block, i.e. (I kron H_b) instead of H_n.
  * Normalisation: 1/sqrt(b) per block, so that the map is orthogonal.

The product is formed with a dense float64 matrix multiply (a library
primitive); nothing is blocked, reordered or fused beyond the definition.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from .hadamard import hadamard


def _block_width(dim: int, block: int) -> int:
    b = dim if block == 0 else block
    if b <= 0 or dim % b != 0:
        raise ValueError(f"block {block} does not divide dim {dim}")
    return b


def _signed(x: np.ndarray, signs: Optional[np.ndarray]) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    if signs is None:
        return x
    s = np.asarray(signs, dtype=np.float64)
    if s.shape != (x.shape[-1],) or not np.all(np.abs(s) == 1.0):
        raise ValueError("signs must be a +-1 vector of length dim")
    return x * s[None, :]


def rht_unnormalized(x: np.ndarray, signs: Optional[np.ndarray],
                     block: int) -> np.ndarray:
    """S = (x . D) . (I kron H_b)^T, without the 1/sqrt(b) factor (float64).

    S_i = sum_j H[i][j] s_j x_j inside each block.  For bf16 inputs every
    product is exact and the float64 sums are exact unless one block spans more
    than about 2^30 in magnitude.
    """
    xs = _signed(x, signs)
    t, n = xs.shape
    b = _block_width(n, block)
    h = hadamard(b)
    s = xs.reshape(t * (n // b), b) @ h.T
    return s.reshape(t, n)


def rht(x: np.ndarray, signs: Optional[np.ndarray], block: int) -> np.ndarray:
    """Forward RHT: y = S / sqrt(b) with IEEE float64 sqrt and division."""
    n = np.asarray(x).shape[-1]
    b = _block_width(n, block)
    return rht_unnormalized(x, signs, block) / np.sqrt(np.float64(b))


def rht_inverse(y: np.ndarray, signs: Optional[np.ndarray],
                block: int) -> np.ndarray:
    """Inverse RHT: x = D . H . y / sqrt(b) per block, i.e.
    x_j = s_j sum_i H[i][j] y_i / sqrt(b) (the transpose of the forward map)."""
    y = np.asarray(y, dtype=np.float64)
    t, n = y.shape
    b = _block_width(n, block)
    h = hadamard(b)
    z = (y.reshape(t * (n // b), b) @ h).reshape(t, n) / np.sqrt(np.float64(b))
    if signs is not None:
        z = z * np.asarray(signs, dtype=np.float64)[None, :]
    return z
