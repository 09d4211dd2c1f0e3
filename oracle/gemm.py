"""The 4-bit GEMM that consumes rotated, NVFP4-quantized activations (oracle,
test infrastructure only).

Sources on the pages:
  * QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs (reviews), review 2
    Strengths and review 4 Strengths: the end-to-end prefill speedup of the
    rotated 4-bit path (">3x", "up to 3.33x") comes from running the
    projections as 4-bit GEMMs on the quantized activations and weights;
    review 4 Questions: the 4-bit GEMM kernels are CUTLASS-based.
  * Same page, review 3 Questions: the Hadamard block computes Y = X H^T, so
    rotating both the activation rows x and the weight rows w by the same
    orthogonal map leaves every product x . w^T unchanged (the rotation is
    "computationally invariant" for the GEMM).
  * Methodology checks for NVFP4 W4A4 on Qwen3-8B (forum thread),
    krylov_schur §3 table: NVFP4 (E2M1 codes, one E4M3 scale per 16
    elements, fp32 tensor scale) for both weights and activations (W4A4).

What it computes.  For A (M x K) and B (N x K), both NVFP4 with their
dequantized values a = E2M1(code) * E4M3(s_b) * t (the definition of
`quant.dequant_nvfp4` before its fp32 rounding):
    C[m][n] = sum_k a[m][k] b[n][k].
Evaluated as (sum_k (E2M1 * E4M3)_a (E2M1 * E4M3)_b) * (t_a * t_b): every
unscaled product has at most 12 significant bits and is exact in float64, the
float64 sum of K of them errs by at most K 2^-53 of the sum of magnitudes,
and t_a * t_b (two fp32 values) is exact in float64; the last product rounds
once.  `nvfp4_gemm_abs` gives sum_k |a[m][k] b[n][k]|, the scale of the
rounding error of any fp32 accumulation of the same products.

Scale-factor layout for a tensor-core consumer.  The pages give no layout for
the block scales (reading r11: row-major and linear).  A tcgen05 block-scaled
MMA reads its scale factors from tensor memory, where one K = 64 step of 128
rows takes a 512-byte atom: 32 lanes of 16 bytes, lane r % 32 holding, at
byte 4 * ((r // 32) % 4) + (c % 4), the scale of row r and 16-block c.  Atoms
follow each other along the 16-block index (c // 4) within a 128-row block,
and row blocks follow each other (the NVIDIA documented "128 x 4" layout of
1-D block-scaling factors).  `sf_mma_layout` writes the linear [rows, kc]
scales in that order, rows padded to a multiple of 128 and kc to a multiple
of 4 with zero bytes; `sf_from_mma_layout` reads them back.  The layout is a
hardware format, not a choice of the method: on the CPU it is pinned as a
bijection with its inverse; on the GPU the tensor core itself checks it (a
GEMM fed scales in any other order disagrees with `nvfp4_gemm`).
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e4m3_decode

NVFP4_BLOCK = 16
SF_ROWS = 128          # rows of one scale-factor atom block
SF_COLS = 4            # 16-blocks per atom (one K = 64 MMA step)
SF_ATOM_BYTES = 512


def _unscaled(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """E2M1(code) * E4M3(s_b) in float64 (exact), [rows, K]."""
    c = np.asarray(codes)
    rows, k = c.shape
    if k % NVFP4_BLOCK:
        raise ValueError("K must be a multiple of 16")
    s = np.asarray(scales)
    if s.shape != (rows, k // NVFP4_BLOCK):
        raise ValueError("block scales must be [rows, K/16]")
    v = e2m1_decode(c).reshape(rows, k // NVFP4_BLOCK, NVFP4_BLOCK)
    return (v * e4m3_decode(s)[..., None]).reshape(rows, k)


def nvfp4_gemm(codes_a, scales_a, ta, codes_b, scales_b, tb) -> np.ndarray:
    """C = dequant(A) . dequant(B)^T, float64 [M, N].  codes: 4-bit E2M1 codes
    (unpacked, one per element), scales: E4M3 codes [rows, K/16] (linear),
    ta / tb: the fp32 tensor scales."""
    ua = _unscaled(codes_a, scales_a)
    ub = _unscaled(codes_b, scales_b)
    if ua.shape[1] != ub.shape[1]:
        raise ValueError("A and B must have the same K")
    return (ua @ ub.T) * (np.float64(np.float32(ta)) * np.float64(np.float32(tb)))


def nvfp4_gemm_abs(codes_a, scales_a, ta, codes_b, scales_b, tb) -> np.ndarray:
    """sum_k |a[m][k] b[n][k]| (float64 [M, N])."""
    ua = np.abs(_unscaled(codes_a, scales_a))
    ub = np.abs(_unscaled(codes_b, scales_b))
    return (ua @ ub.T) * abs(np.float64(np.float32(ta)) * np.float64(np.float32(tb)))


def _padded(rows: int, kc: int):
    return -(-rows // SF_ROWS) * SF_ROWS, -(-kc // SF_COLS) * SF_COLS


def sf_mma_layout(scales: np.ndarray) -> np.ndarray:
    """Linear block scales [rows, kc] -> the tensor-core scale-factor layout,
    a flat uint8 array of padded_rows * padded_kc bytes (zero padding)."""
    s = np.asarray(scales, dtype=np.uint8)
    rows, kc = s.shape
    pr, pk = _padded(rows, kc)
    p = np.zeros((pr, pk), dtype=np.uint8)
    p[:rows, :kc] = s
    # [row block, r1 = (r // 32) % 4, r0 = r % 32, atom column c // 4, c % 4]
    t = p.reshape(pr // SF_ROWS, 4, 32, pk // SF_COLS, SF_COLS)
    # atom order: row block, then atom column; inside: r0 (16 bytes each), r1, c % 4
    return np.ascontiguousarray(t.transpose(0, 3, 2, 1, 4)).reshape(-1)


def sf_from_mma_layout(flat: np.ndarray, rows: int, kc: int) -> np.ndarray:
    """Inverse of sf_mma_layout: the linear [rows, kc] scales."""
    pr, pk = _padded(rows, kc)
    f = np.asarray(flat, dtype=np.uint8)
    if f.size != pr * pk:
        raise ValueError("size does not match the padded layout")
    t = f.reshape(pr // SF_ROWS, pk // SF_COLS, 32, 4, SF_COLS)
    return np.ascontiguousarray(t.transpose(0, 3, 2, 1, 4)).reshape(pr, pk)[:rows, :kc]
