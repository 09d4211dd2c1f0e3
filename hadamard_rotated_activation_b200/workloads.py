"""Seeded synthetic activations for the five reference workloads.

This module only draws random numbers and rounds them to the storage type of
the workload (bf16 with round-to-nearest-even, or fp32).  It holds none of the
rotation or quantization arithmetic: the CUDA path and the CPU oracle both take
their inputs from here and share nothing else.

The value distributions stand in for the activation statistics the pages
describe: outlier channels (QuaRot reviews, review 3 summary: "outlier
features in activations"), attention-sink tokens whose RMS is 30-50x the
ordinary tokens on fewer than 0.5% of rows ("Methodology checks for NVFP4 W4A4
on Qwen3-8B" thread, krylov_schur §1 "Attention-Sink Effective Sample
Collapse"), and the Qwen3-8B shapes hidden 4096 / intermediate 12288
("Bug: Qwen3-8B integration issue", Model Details table).  No public dataset is
used.

Draw order per workload (fixed, so a seed names one input):
  signs -> outlier / sink index choice -> per-channel or per-head scales ->
  entries.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

# storage types
F32 = "f32"
BF16 = "bf16"

# output formats
INT4_SYM = "int4_sym"
INT4_ASYM = "int4_asym"
NVFP4 = "nvfp4"


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shape, storage type, rotation and output format."""

    key: str
    tokens: int
    dim: int
    dtype: str
    block: int          # 0 = Hadamard over the full row, else the block width
    use_signs: bool     # random +-1 diagonal D before H
    fmt: str
    seed: int
    group: int = 0      # asymmetric INT4 group size (0 = per token)
    heads: int = 0      # KV-cache view: dim = heads * head_dim
    description: str = ""

    @property
    def elements(self) -> int:
        return self.tokens * self.dim

    def with_tokens(self, tokens: int) -> "Workload":
        return replace(self, tokens=int(tokens))

    def algorithmic_bytes(self) -> int:
        """One read of the input plus one write of codes and scales.

        Signs and the 4-byte tensor scale are counted too (they are tiny).
        """
        t, n = self.tokens, self.dim
        elt = 4 if self.dtype == F32 else 2
        rd = t * n * elt + (n if self.use_signs else 0)
        codes = t * n // 2
        if self.fmt == INT4_SYM:
            scales = 4 * t
        elif self.fmt == INT4_ASYM:
            scales = 2 * 2 * t * (n // self.group)
        else:  # NVFP4: one E4M3 byte per 16 elements + fp32 tensor scale
            scales = t * n // 16 + 4
        return rd + codes + scales


WORKLOADS = {
    "c1": Workload(
        "c1", 64, 4096, F32, 0, True, INT4_SYM, seed=0,
        description="64 tokens x 4096 fp32, N(0,1) with 8 outlier channels x50; "
                    "full-4096 RHT; per-token symmetric INT4"),
    "c2": Workload(
        "c2", 2048, 4096, BF16, 128, True, NVFP4, seed=1,
        description="2048 x 4096 bf16, N(0,1) x lognormal(0,1) per channel, 1% "
                    "outlier channels x30; block-128 RHT; NVFP4, dynamic tensor scale"),
    "c3": Workload(
        "c3", 2048, 12288, BF16, 0, True, INT4_SYM, seed=2,
        description="2048 x 12288 bf16 (down_proj input), Student-t nu=3, 0.5% "
                    "sink rows x40; H12 (Paley) x H1024 RHT; per-token symmetric INT4"),
    "c4": Workload(
        "c4", 16384, 4096, BF16, 0, True, NVFP4, seed=3,
        description="16384 x 4096 bf16 (8 x 2048 batch), N(0,1) x lognormal(0,1.5) "
                    "per channel; full-4096 RHT; NVFP4; dequant + inverse round trip"),
    "c5": Workload(
        "c5", 32768, 4096, BF16, 128, False, INT4_ASYM, seed=4, group=128, heads=32,
        description="KV cache 32768 tokens x 32 heads x 128 bf16, N(0,1) x "
                    "lognormal(0,1) per head, 2 outlier dims per head x20; per-head "
                    "H128, no signs; asymmetric INT4 g128 (fp16 scale + zero)"),
}


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits) with ties to even.

    Returns float64 values that are exactly representable in bf16.  Rounds in
    one step from float64 (no double rounding through float32).  The workloads
    stay far inside the bf16 normal range.
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2**e, 0.5 <= |m| < 1
    r = np.rint(np.ldexp(m, 8))             # 8 significant bits, ties to even
    out = np.ldexp(r, e - 8)
    if not np.all(np.isfinite(out)):
        raise ValueError("value outside the bf16 range")
    tiny = (out != 0) & (np.abs(out) < 2.0 ** -126)
    if np.any(tiny):
        raise ValueError("value in the bf16 subnormal range")
    return out


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of values that are already bf16-representable."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    """float64 values of uint16 bf16 bit patterns (exact widening)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


@dataclass
class Inputs:
    """Host-side input of one workload.

    values: float64 [tokens, dim], exactly the stored values (bf16 or fp32).
    stored: the array handed to the device: uint16 bf16 bits or float32.
    signs:  int8 [dim] of +-1, or None.
    """

    workload: Workload
    values: np.ndarray
    stored: np.ndarray
    signs: Optional[np.ndarray]


def _choice(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    return np.sort(rng.choice(n, size=k, replace=False))


def make_inputs(w: Workload, tokens: Optional[int] = None,
                seed: Optional[int] = None) -> Inputs:
    """Draw the input of workload `w` (optionally with another row count/seed)."""
    if tokens is not None:
        w = w.with_tokens(tokens)
    if seed is not None:
        w = replace(w, seed=int(seed))
    rng = np.random.default_rng(w.seed)
    t, n = w.tokens, w.dim

    signs = None
    if w.use_signs:
        signs = (1 - 2 * rng.integers(0, 2, size=n)).astype(np.int8)

    if w.key == "c1":
        outl = _choice(rng, n, 8)
        x = rng.standard_normal((t, n))
        x[:, outl] *= 50.0
    elif w.key == "c2":
        outl = _choice(rng, n, int(round(0.01 * n)))
        c = rng.lognormal(0.0, 1.0, size=n)
        c[outl] *= 30.0
        x = rng.standard_normal((t, n)) * c[None, :]
    elif w.key == "c3":
        k = max(1, int(round(0.005 * t)))
        sinks = _choice(rng, t, k)
        x = rng.standard_t(3.0, size=(t, n))
        x[sinks, :] *= 40.0
    elif w.key == "c4":
        c = rng.lognormal(0.0, 1.5, size=n)
        x = rng.standard_normal((t, n)) * c[None, :]
    elif w.key == "c5":
        h = w.heads
        hd = n // h
        outl = np.stack([_choice(rng, hd, 2) for _ in range(h)])  # [h, 2]
        c = rng.lognormal(0.0, 1.0, size=h)
        scale = np.repeat(c, hd)
        for hh in range(h):
            scale[hh * hd + outl[hh]] *= 20.0
        x = rng.standard_normal((t, n)) * scale[None, :]
    else:
        raise KeyError(w.key)

    if w.dtype == BF16:
        vals = round_to_bf16(x)
        stored = bf16_bits(vals)
    else:
        stored = x.astype(np.float32)
        vals = stored.astype(np.float64)
    return Inputs(w, vals, stored, signs)


def edge_rows(dim: int, dtype: str, rng_seed: int = 7) -> np.ndarray:
    """A few degenerate rows: zeros, one spike, all equal, tiny and huge values.

    Used by the edge-case parity tests.  Returned as float64 values that are
    representable in `dtype`.
    """
    rng = np.random.default_rng(rng_seed)
    rows = []
    rows.append(np.zeros(dim))
    spike = np.zeros(dim)
    spike[dim // 3] = 3.5
    rows.append(spike)
    rows.append(np.full(dim, 0.75))
    alt = np.where(np.arange(dim) % 2 == 0, 1.0, -1.0)
    rows.append(alt)
    rows.append(rng.standard_normal(dim) * 1e-3)
    big = rng.standard_normal(dim)
    big[::97] *= 1e4
    rows.append(big)
    x = np.stack(rows)
    if dtype == BF16:
        return round_to_bf16(x)
    return x.astype(np.float32).astype(np.float64)


@dataclass
class CodedInputs:
    """Host-side input of a dequantizing call: packed codes and their scales.

    codes:  uint8 [tokens, dim/2], two 4-bit codes per byte (low nibble first).
    scales: fp32 [tokens] (INT4 symmetric), fp16 [tokens, dim/group]
            (asymmetric) or E4M3 bytes [tokens, dim/16] (NVFP4).
    zeros:  fp16 [tokens, dim/group] (asymmetric) or None.
    tensor_scale: fp32 (NVFP4) or None.
    signs:  int8 [dim] of +-1, or None.
    """

    workload: Workload
    codes: np.ndarray
    scales: np.ndarray
    zeros: Optional[np.ndarray]
    tensor_scale: Optional[np.float32]
    signs: Optional[np.ndarray]


def make_coded_inputs(w: Workload, tokens: Optional[int] = None,
                      seed: Optional[int] = None) -> CodedInputs:
    """Uniformly random codes and scales in the format of workload `w`.

    Every 4-bit code value is equally likely.  NVFP4 block scales are uniform
    over the finite E4M3 codes 0x00..0x7E (zero and subnormal scales
    included); the tensor scale is fixed at 2^-8 * 1.37.  INT4 scales are
    lognormal; asymmetric zeros are uniform on [0, 15] in fp16.  The signs are
    those `make_inputs` draws for the same workload.
    """
    if tokens is not None:
        w = w.with_tokens(tokens)
    t, n = w.tokens, w.dim
    signs = make_inputs(w, tokens=1).signs
    rng = np.random.default_rng(1000 + (w.seed if seed is None else int(seed)))
    codes = rng.integers(0, 256, size=(t, n // 2), dtype=np.uint8)
    zeros = None
    tscale = None
    if w.fmt == NVFP4:
        scales = rng.integers(0, 0x7F, size=(t, n // 16), dtype=np.uint8)
        tscale = np.float32(1.37 * 2.0 ** -8)
    elif w.fmt == INT4_SYM:
        scales = rng.lognormal(-2.0, 1.0, size=t).astype(np.float32)
    else:
        scales = rng.lognormal(-3.0, 1.0, size=(t, n // w.group)).astype(np.float16)
        zeros = rng.uniform(0.0, 15.0, size=(t, n // w.group)).astype(np.float16)
    return CodedInputs(w, codes, scales, zeros, tscale, signs)
