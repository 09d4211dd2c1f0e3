"""Small number formats used by the quantizers (oracle, test infrastructure only).

The pages name the formats but do not define them bit for bit:
  * Methodology checks for NVFP4 W4A4 on Qwen3-8B (forum thread), krylov_schur
    §3 table: NVFP4 costs 4.50 bits per element (4-bit code + one 8-bit scale
    per 16 elements).
  * Same thread, discrete_descent's reply: deterministic FP4 rounding flushes
    small values to zero.
The bit-level definitions below follow the public format specifications:
  * E2M1 (FP4): OCP Microscaling Formats (MX) v1.0, the FP4 element type:
    1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no Inf/NaN.
  * E4M3 (FP8): OCP 8-bit Floating Point (OFP8) specification, E4M3:
    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no Inf,
    S.1111.111 is NaN, largest finite 448, smallest subnormal 2^-9.
  * fp16: IEEE 754 binary16 (numpy's float16 conversion, pinned by a test
    against a brute-force nearest search).

Encoders search every finite code for the nearest value, ties going to the
code with an even mantissa bit (round to nearest even), and saturate to the
largest finite magnitude (the "satfinite" reading).
"""
from __future__ import annotations

import numpy as np


def _e2m1_magnitude(idx: int) -> float:
    """Magnitude of the 3-bit E2M1 field idx = (exponent << 1) | mantissa."""
    e, m = idx >> 1, idx & 1
    if e == 0:
        return m * 0.5                     # subnormal: m * 2^(1-bias) / 2
    return (1.0 + m / 2.0) * 2.0 ** (e - 1)


E2M1_GRID = np.array([_e2m1_magnitude(i) for i in range(8)])  # 0 .. 6


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    """Value of 4-bit E2M1 codes (bit 3 = sign, bits 0-2 = magnitude index)."""
    c = np.asarray(code, dtype=np.int64)
    mag = E2M1_GRID[c & 7]
    return np.where((c & 8) != 0, -mag, mag)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """Round float64 values to E2M1 codes: nearest, ties to even index, satfinite.

    Sign bit = (v < 0), so a negative value that rounds to zero gives 0x8.
    Elementwise; processed in chunks only to bound memory.
    """
    v = np.asarray(v, dtype=np.float64)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    chunk = 1 << 20
    for s in range(0, flat.size, chunk):
        x = flat[s:s + chunk]
        a = np.abs(x)
        d = np.abs(a[:, None] - E2M1_GRID[None, :])          # distance to each code
        best = np.min(d, axis=1, keepdims=True)
        tie = d == best
        # among equally near codes take the even index; at most two can tie
        even = tie & ((np.arange(8) & 1) == 0)[None, :]
        idx = np.where(np.any(even, axis=1), np.argmax(even, axis=1),
                       np.argmax(tie, axis=1))
        idx = np.where(a >= E2M1_GRID[7], 7, idx)             # saturate
        sign = (x < 0).astype(np.int64) << 3
        out[s:s + chunk] = idx.astype(np.int64) | sign
    return out.reshape(v.shape)


def _e4m3_value(code: int) -> float:
    s, e, m = (code >> 7) & 1, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        mag = m * 2.0 ** -9                                # subnormal
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)])
_E4M3_POS = E4M3_TABLE[:127]          # codes 0x00 .. 0x7E, all finite, >= 0


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(code, dtype=np.int64) & 0xFF]


def e4m3_encode(r: np.ndarray) -> np.ndarray:
    """Round non-negative values to E4M3 codes: nearest, ties to even, satfinite.

    Input values are finite and >= 0 (block scales).  Values above 448 give
    0x7E (448).
    """
    r = np.asarray(r, dtype=np.float64)
    if np.any(~np.isfinite(r)) or np.any(r < 0):
        raise ValueError("E4M3 scale input must be finite and non-negative")
    flat = r.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    chunk = 1 << 16
    codes = np.arange(127)
    for s in range(0, flat.size, chunk):
        a = flat[s:s + chunk]
        d = np.abs(a[:, None] - _E4M3_POS[None, :])
        best = np.min(d, axis=1, keepdims=True)
        tie = d == best
        even = tie & ((codes & 1) == 0)[None, :]
        idx = np.where(np.any(even, axis=1), np.argmax(even, axis=1),
                       np.argmax(tie, axis=1))
        idx = np.where(a >= _E4M3_POS[126], 126, idx)
        out[s:s + chunk] = idx
    return out.reshape(r.shape)


def fp16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 to IEEE binary16 in one step (numpy float16 conversion)."""
    return np.asarray(v, dtype=np.float64).astype(np.float16)
