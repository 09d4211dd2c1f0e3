"""Scalar 4-bit quantizers and dequantizers (oracle, test infrastructure only).

Sources on the pages:
  * QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs (reviews), review 2
    Summary and Weaknesses: after the RHT the activations are quantized with
    round-to-nearest (RTN) to INT4, symmetric, with one scale per token.
  * Same page, review 2 final comments and review 3 Summary: W4A4KV4, the KV
    cache at 4 bits per 128-dim head; Methodology checks for NVFP4 W4A4 on
    Qwen3-8B (forum thread), discrete_descent's note: INT4-g128 (group-128
    INT4).  Read here as asymmetric INT4, fp16 scale and fp16 integer
    zero-point per group of 128.
  * Same forum thread, krylov_schur §3 table: NVFP4 at 4.50 bits per element,
    i.e. E2M1 codes with one E4M3 scale per 16 elements; the per-tensor fp32
    scale is amax / (6 * 448) (6 = largest E2M1, 448 = largest E4M3).

Readings where the pages are silent (each listed in the design notes):
  * INT4 symmetric: scale32 = fp32(amax64 / 7); q = clamp(rint(y / scale32),
    -8, 7) with ties to even; a zero row has scale 0 and codes 0.
  * NVFP4: t = fp32(g64 / 2688) for the dynamic tensor scale, or the caller's
    t (static); per 16-block r = fp32(b64 / (6 t)), s_b = E4M3(r) (nearest even,
    satfinite); v = y / (E4M3value(s_b) * t) (exact product in float64);
    code = E2M1(v), sign bit = (y < 0).  When E4M3value(s_b) * t is 0 every
    code of the block is 0 with the sign bit of y.
  * INT4 asymmetric: scale16 = fp16((mx - mn) / 15) in one rounding;
    z = rint(-mn / scale16), stored as fp16; u = clamp(rint(y / scale16) + z,
    0, 15) using the stored z; a group with scale16 == 0 has z = 0, u = 0.
  * MXFP4 (named on the same thread, discrete_descent's comparison of
    rotations under NVFP4, MXFP4 and INT4-g128; the pages give no bit-level
    definition): the public OCP Microscaling Formats (MX) v1.0 reading.
    Blocks of 32 consecutive elements share an E8M0 scale X = 2^e with
    e = floor(log2(amax64)) - 2 (2 = the largest E2M1 exponent), clamped to
    [-127, 127], stored as the byte e + 127; an all-zero block has e = -127.
    code = E2M1(y / X) (nearest even, saturating at 6), sign bit = (y < 0).
  * Dequantization: the exact product of code and scale(s), rounded once to
    fp32.
  * Packing: two codes per byte, element 2k in bits 0-3, 2k+1 in bits 4-7.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .formats import (
    e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, fp16_round,
)

E2M1_MAX = 6.0
E4M3_MAX = 448.0


# ----------------------------------------------------------------- packing
def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., n] 4-bit codes (0..15 or two's-complement INT4) -> [..., n/2] bytes."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    if c.shape[-1] % 2:
        raise ValueError("odd number of codes")
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """[..., n/2] bytes -> [..., n] 4-bit codes 0..15 (low nibble first)."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def int4_from_nibble(nib: np.ndarray) -> np.ndarray:
    """Two's-complement nibble 0..15 -> -8..7."""
    n = np.asarray(nib, dtype=np.int64)
    return np.where(n >= 8, n - 16, n)


# ------------------------------------------------------ INT4, per token
def int4_sym_per_token(y: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-token symmetric INT4 of rotated rows y (float64 [T, n]).

    Returns (q int64 [T, n] in -8..7, scale float32 [T]).
    """
    y = np.asarray(y, dtype=np.float64)
    amax = np.max(np.abs(y), axis=1)
    scale = (amax / 7.0).astype(np.float32)
    s64 = scale.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.clip(np.rint(y / s64), -8, 7)
    q = np.where(s64 > 0, q, 0.0)
    return q.astype(np.int64), scale


def dequant_int4_sym(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    q = np.asarray(q, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)[:, None]
    return (q * s).astype(np.float32)


# --------------------------------------------- INT4 asymmetric, per group
def int4_asym_group(y: np.ndarray, group: int
                    ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Asymmetric INT4 per group of `group` consecutive elements of a row.

    Returns (u int64 [T, n] in 0..15, scale fp16 [T, n/group],
    zero fp16 [T, n/group]).
    """
    y = np.asarray(y, dtype=np.float64)
    t, n = y.shape
    if n % group:
        raise ValueError("group does not divide dim")
    g = y.reshape(t, n // group, group)
    mx = np.max(g, axis=2)
    mn = np.min(g, axis=2)
    scale16 = fp16_round((mx - mn) / 15.0)
    s64 = scale16.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(s64 > 0, np.rint(-mn / s64), 0.0)
    z16 = fp16_round(z)
    z64 = z16.astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.clip(np.rint(g / s64[..., None]) + z64[..., None], 0, 15)
    u = np.where(s64[..., None] > 0, u, 0.0)
    return u.reshape(t, n).astype(np.int64), scale16, z16


def dequant_int4_asym(u: np.ndarray, scale16: np.ndarray, zero16: np.ndarray,
                      group: int) -> np.ndarray:
    u = np.asarray(u, dtype=np.float64)
    t, n = u.shape
    s = np.asarray(scale16, dtype=np.float16).astype(np.float64)
    z = np.asarray(zero16, dtype=np.float16).astype(np.float64)
    g = u.reshape(t, n // group, group)
    return (s[..., None] * (g - z[..., None])).reshape(t, n).astype(np.float32)


# ------------------------------------------------------------------ NVFP4
def nvfp4_tensor_scale(y: np.ndarray) -> np.float32:
    """Dynamic tensor scale t = fp32(amax(|y|) / (6 * 448))."""
    g = np.max(np.abs(np.asarray(y, dtype=np.float64)))
    return np.float32(g / (E2M1_MAX * E4M3_MAX))


def nvfp4(y: np.ndarray, tensor_scale: Optional[float] = None
          ) -> Tuple[np.ndarray, np.ndarray, np.float32]:
    """NVFP4 of rotated rows y (float64 [T, n], n % 16 == 0).

    Returns (codes uint8 [T, n] E2M1 4-bit codes, block_scales uint8
    [T, n/16] E4M3 codes, tensor_scale float32).
    """
    y = np.asarray(y, dtype=np.float64)
    t_rows, n = y.shape
    if n % 16:
        raise ValueError("NVFP4 needs dim % 16 == 0")
    t = nvfp4_tensor_scale(y) if tensor_scale is None else np.float32(tensor_scale)
    t64 = np.float64(t)
    blk = y.reshape(t_rows, n // 16, 16)
    bmax = np.max(np.abs(blk), axis=2)
    if t64 > 0:
        r = (bmax / (E2M1_MAX * t64)).astype(np.float32)
    else:
        r = np.zeros_like(bmax, dtype=np.float32)
    sb = e4m3_encode(r.astype(np.float64))
    denom = e4m3_decode(sb) * t64                     # exact in float64
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(denom[..., None] > 0, blk / denom[..., None], 0.0)
    codes = e2m1_encode(v)
    # blocks with a zero denominator keep only the sign of y
    zero_den = np.broadcast_to(denom[..., None] <= 0, blk.shape)
    codes = np.where(zero_den, (blk < 0).astype(np.uint8) << 3, codes)
    return codes.reshape(t_rows, n).astype(np.uint8), sb, t


def dequant_nvfp4(codes: np.ndarray, block_scales: np.ndarray,
                  tensor_scale: float) -> np.ndarray:
    c = np.asarray(codes)
    t_rows, n = c.shape
    v = e2m1_decode(c).reshape(t_rows, n // 16, 16)
    s = e4m3_decode(block_scales)[..., None] * np.float64(np.float32(tensor_scale))
    return (v * s).reshape(t_rows, n).astype(np.float32)


# ------------------------------------------------------------------ MXFP4
MX_BLOCK = 32
E2M1_EMAX = 2          # largest E2M1 value 6 = 1.5 * 2^2


def mxfp4_exponents(y: np.ndarray) -> np.ndarray:
    """Shared exponent e per 32-block of rows y (float64 [T, n]), int64
    [T, n/32]: floor(log2(max |y|)) - 2 clamped to [-127, 127] (frexp gives
    floor(log2) exactly); an all-zero block gets -127."""
    y = np.asarray(y, dtype=np.float64)
    t_rows, n = y.shape
    if n % MX_BLOCK:
        raise ValueError("MXFP4 needs dim % 32 == 0")
    amax = np.max(np.abs(y.reshape(t_rows, n // MX_BLOCK, MX_BLOCK)), axis=2)
    _, ex = np.frexp(amax)                      # amax = m 2^ex, 0.5 <= m < 1
    e = ex.astype(np.int64) - 1 - E2M1_EMAX
    e = np.where(amax > 0, e, -127)
    return np.clip(e, -127, 127)


def mxfp4(y: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """MXFP4 of rotated rows y (float64 [T, n], n % 32 == 0).

    Returns (codes uint8 [T, n] E2M1 4-bit codes, scales uint8 [T, n/32]
    E8M0 bytes e + 127).
    """
    y = np.asarray(y, dtype=np.float64)
    t_rows, n = y.shape
    e = mxfp4_exponents(y)
    blk = y.reshape(t_rows, n // MX_BLOCK, MX_BLOCK)
    v = blk / np.ldexp(1.0, e)[..., None]       # exact: division by a power of two
    codes = e2m1_encode(v)
    return codes.reshape(t_rows, n).astype(np.uint8), (e + 127).astype(np.uint8)


def dequant_mxfp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    c = np.asarray(codes)
    t_rows, n = c.shape
    v = e2m1_decode(c).reshape(t_rows, n // MX_BLOCK, MX_BLOCK)
    x = np.ldexp(1.0, np.asarray(scales, dtype=np.int64) - 127)[..., None]
    with np.errstate(over="ignore"):
        return (v * x).reshape(t_rows, n).astype(np.float32)
