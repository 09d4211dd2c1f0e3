"""Comparison helpers: CUDA path (through the C ABI) vs the CPU oracle.

Criteria (from the parity contract of the method):
  * rotated fp32 values: relative L2 error per row <= 2e-6; an all-zero row
    must come out exactly zero;
  * scales (fp32 per token, fp16 scale/zero, E4M3 block scale, fp32 tensor
    scale): bit-exact;
  * packed 4-bit codes: bit-exact, except where the oracle's value before
    rounding lies within 1e-5 (relative) of a rounding boundary; those cases
    are counted and returned, not hidden.  For NVFP4 the sign bit of a code
    whose magnitude rounds to zero is decided at 0, which is treated as a
    boundary with an absolute window of 1e-5 in code units.
  * dequantized values: bit-exact (the GPU's codes and scales fed to the
    oracle's dequantizer).
"""
from __future__ import annotations

import functools
import os
from dataclasses import asdict, astuple, dataclass

import numpy as np
import torch

import oracle
from oracle.quant import int4_from_nibble
from hadamard_rotated_activation_b200 import workloads as wl
import hadamard_rotated_activation_b200 as kq

REL_L2 = 2e-6
NEAR = 1e-5
E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


# ------------------------------------------------------------ device I/O
def to_device(inp: wl.Inputs, device="cuda"):
    w = inp.workload
    if w.dtype == wl.BF16:
        x = torch.from_numpy(inp.stored.view(np.int16)).to(device).view(torch.bfloat16)
    else:
        x = torch.from_numpy(inp.stored).to(device)
    s = None if inp.signs is None else torch.from_numpy(inp.signs).to(device)
    return x, s


def stored_from_values(values: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == wl.BF16:
        return wl.bf16_bits(values)
    return values.astype(np.float32)


def inputs_from_values(w: wl.Workload, values: np.ndarray, signs) -> wl.Inputs:
    return wl.Inputs(w.with_tokens(values.shape[0]), values,
                     stored_from_values(values, w.dtype), signs)


# ---------------------------------------------------------- GPU runners
def gpu_rht(inp: wl.Inputs, inverse=False, x_override=None):
    w = inp.workload
    x, s = to_device(inp)
    if x_override is not None:
        x = x_override
    out = torch.empty((x.shape[0], w.dim), dtype=torch.float32, device=x.device)
    kq.kq_rht(x, w.block, s, out, inverse=inverse)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_int4_sym(inp: wl.Inputs):
    w = inp.workload
    x, s = to_device(inp)
    codes, scales = kq.empty_int4_sym(w.tokens, w.dim)
    kq.kq_rht_quant_int4(x, w.block, s, 0, False, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def gpu_int4_asym(inp: wl.Inputs, group=128):
    w = inp.workload
    x, s = to_device(inp)
    codes, scales, zeros = kq.empty_int4_asym(w.tokens, w.dim, group)
    kq.kq_rht_quant_int4(x, w.block, s, group, True, codes, scales, zeros)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), zeros.cpu().numpy()


def gpu_nvfp4(inp: wl.Inputs, tensor_scale=None):
    """Dynamic tensor scale when tensor_scale is None, else static."""
    w = inp.workload
    x, s = to_device(inp)
    codes, bs, ts, ws = kq.empty_nvfp4(w.tokens, w.dim, w.block)
    if tensor_scale is None:
        kq.kq_rht_quant_nvfp4(x, w.block, s, codes, bs, ts, ws, dynamic=True)
    else:
        ts.fill_(float(np.float32(tensor_scale)))
        kq.kq_rht_quant_nvfp4(x, w.block, s, codes, bs, ts, None, dynamic=False)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), bs.cpu().numpy(), np.float32(ts.cpu().numpy()[0])


def gpu_dequant(fmt, codes, scales, zeros, tensor_scale, tokens, dim, group=0):
    dev = "cuda"
    c = torch.from_numpy(np.ascontiguousarray(codes)).to(dev)
    if fmt == kq.KQ_FMT_INT4_SYM:
        s = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
        z = None
        t = None
    elif fmt == kq.KQ_FMT_INT4_ASYM:
        s = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
        z = torch.from_numpy(np.ascontiguousarray(zeros)).to(dev)
        t = None
    elif fmt == kq.KQ_FMT_MXFP4:
        s = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
        z = None
        t = None
    else:
        s = torch.from_numpy(np.ascontiguousarray(scales)).to(dev)
        z = None
        t = torch.tensor([float(tensor_scale)], dtype=torch.float32, device=dev)
    out = torch.empty((tokens, dim), dtype=torch.float32, device=dev)
    kq.kq_dequant(fmt, c, s, z, t, tokens, dim, group, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_dequant_rht_inverse(ci: wl.CodedInputs, signs_mode: str = "aligned",
                            out_dtype: str = "f32"):
    """kq_dequant_rht_inverse on coded inputs.  signs_mode: "aligned" (the
    signs at a 16-byte boundary), "offset8" (8 bytes past one: a call the
    tensor-core kernel declines), or "none" (no signs)."""
    w = ci.workload
    dev = "cuda"
    c = torch.from_numpy(np.ascontiguousarray(ci.codes)).to(dev)
    s = torch.from_numpy(np.ascontiguousarray(ci.scales)).to(dev)
    z = None if ci.zeros is None else torch.from_numpy(np.ascontiguousarray(ci.zeros)).to(dev)
    t = None
    if ci.tensor_scale is not None:
        t = torch.tensor([float(ci.tensor_scale)], dtype=torch.float32, device=dev)
    sg = None
    if ci.signs is not None and signs_mode != "none":
        if signs_mode == "aligned":
            sg = torch.from_numpy(ci.signs).to(dev)
        else:
            buf = torch.zeros(w.dim + 16, dtype=torch.int8, device=dev)
            buf[8:8 + w.dim] = torch.from_numpy(ci.signs).to(dev)
            sg = buf[8:8 + w.dim]
            assert sg.data_ptr() % 16 == 8
    fmt = {wl.INT4_SYM: kq.KQ_FMT_INT4_SYM, wl.INT4_ASYM: kq.KQ_FMT_INT4_ASYM,
           wl.NVFP4: kq.KQ_FMT_NVFP4, "mxfp4": kq.KQ_FMT_MXFP4}[w.fmt]
    tdt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = torch.empty((w.tokens, w.dim), dtype=tdt, device=dev)
    kq.kq_dequant_rht_inverse(fmt, c, s, z, t, w.tokens, w.dim, w.block, w.group, sg, out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def check_rotation_bf16(got: np.ndarray, want: np.ndarray) -> None:
    """bf16 outputs of an fp32 rotation rounded to nearest even.  The fp32
    value lies within tol = REL_L2 * ||row|| of the exact one (the per-row
    criterion bounds every element by the row's error norm); its bf16
    rounding moves it by at most half a bf16 ulp at its own magnitude, which
    is at most |exact| + tol.  An all-zero row must come out exactly zero."""
    got = got.astype(np.float64)
    norm = np.linalg.norm(want, axis=1, keepdims=True)
    tol = REL_L2 * norm
    mag = np.abs(want) + tol
    with np.errstate(divide="ignore"):
        half_ulp = np.where(mag > 0, np.ldexp(1.0, np.frexp(np.where(mag > 0, mag, 1.0))[1] - 9),
                            0.0)
    bad = np.abs(got - want) > half_ulp + tol
    assert not bad.any(), f"{int(bad.sum())} bf16 outputs off by more than half an ulp + tol"
    assert np.all(got[norm[:, 0] == 0] == 0)


def oracle_dequant_rht_inverse(ci: wl.CodedInputs, rows=None, use_signs=True):
    """The oracle's dequantized values (fp32, as kq_dequant defines them),
    rotated back in float64."""
    w = ci.workload
    sel = slice(None) if rows is None else rows
    codes = oracle.unpack_nibbles(ci.codes[sel])
    if w.fmt == wl.NVFP4:
        deq = oracle.dequant_nvfp4(codes, ci.scales[sel], ci.tensor_scale)
    elif w.fmt == wl.INT4_SYM:
        deq = oracle.dequant_int4_sym(int4_from_nibble(codes), ci.scales[sel])
    else:
        deq = oracle.dequant_int4_asym(codes, ci.scales[sel], ci.zeros[sel], w.group)
    signs = ci.signs if use_signs else None
    return oracle.rht_inverse(deq.astype(np.float64), signs, w.block)


# ------------------------------------------------------------ comparisons
def check_rotation(got: np.ndarray, want: np.ndarray) -> float:
    """Max relative L2 error per row; asserts the contract."""
    err = np.linalg.norm(got.astype(np.float64) - want, axis=1)
    ref = np.linalg.norm(want, axis=1)
    zero = ref == 0
    assert np.all(err[zero] == 0), "zero rows must rotate to exact zeros"
    rel = np.where(zero, 0.0, err / np.where(zero, 1.0, ref))
    assert rel.max() <= REL_L2, f"rel L2 {rel.max():.3e} > {REL_L2}"
    return float(rel.max())


def _near_half_integer(v: np.ndarray) -> np.ndarray:
    b = np.floor(v) + 0.5
    return np.abs(v - b) <= NEAR * np.abs(b)


# ------------------------------------------------------- parity counts
@dataclass
class Counts:
    """What one comparison saw.  `scale_mismatch` and `bad` must be zero;
    `near` counts code differences inside the 1e-5 boundary window (allowed,
    and reported rather than hidden)."""
    rows: int = 0
    codes: int = 0
    scales: int = 0
    scale_mismatch: int = 0
    near: int = 0
    bad: int = 0

    def __add__(self, o: "Counts") -> "Counts":
        return Counts(*(a + b for a, b in zip(astuple(self), astuple(o))))

    def as_dict(self) -> dict:
        return asdict(self)


# Every comparison a test makes is added here under a name; conftest prints
# the table at the end of the session (and writes it as JSON when the
# environment variable KQ_PARITY_REPORT names a file).
REPORT: "dict[str, Counts]" = {}


def record(name: str, c: Counts) -> Counts:
    REPORT[name] = REPORT.get(name, Counts()) + c
    return c


def _current_test() -> str:
    """The running test's id without its file, e.g. "test_x[c4-37]"."""
    t = os.environ.get("PYTEST_CURRENT_TEST", "(outside pytest)")
    return t.split("::")[-1].split(" ")[0]


def _finish(c: Counts, strict: bool, what: str, got=None, want=None, mask=None,
            name=None) -> Counts:
    if name is not False:
        record(name or _current_test(), c)
    if strict:
        assert c.scale_mismatch == 0, f"{what}: {c.scale_mismatch} scale mismatches"
        assert c.bad == 0, _first_diff(got, want, what, mask)
    return c


def check_int4_sym(codes, scales, y64, strict=True, name=None) -> Counts:
    """Scales bit for bit; codes bit for bit except near a rounding boundary."""
    q_ref, s_ref = oracle.int4_sym_per_token(y64)
    sm = scales.view(np.uint32) != s_ref.view(np.uint32)
    if strict:
        assert not sm.any(), _first_diff(scales.view(np.uint32), s_ref.view(np.uint32), "scale")
    q = int4_from_nibble(oracle.unpack_nibbles(codes))
    diff = q != q_ref
    s64 = s_ref.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s64 > 0, y64 / s64, 0.0)
    near = _near_half_integer(v)
    bad = diff & ~near
    c = Counts(rows=q.shape[0], codes=q.size, scales=s_ref.size, scale_mismatch=int(sm.sum()),
               near=int((diff & near).sum()), bad=int(bad.sum()))
    return _finish(c, strict, "int4 code", q, q_ref, bad, name)


def check_int4_asym(codes, scales, zeros, y64, group=128, strict=True, name=None) -> Counts:
    u_ref, s_ref, z_ref = oracle.int4_asym_group(y64, group)
    sm = scales.view(np.uint16) != s_ref.view(np.uint16)
    zm = zeros.view(np.uint16) != z_ref.view(np.uint16)
    if strict:
        assert not sm.any(), _first_diff(scales.view(np.uint16), s_ref.view(np.uint16),
                                         "fp16 scale")
        assert not zm.any(), _first_diff(zeros.view(np.uint16), z_ref.view(np.uint16),
                                         "fp16 zero")
    u = oracle.unpack_nibbles(codes)
    diff = u != u_ref
    s = np.repeat(s_ref.astype(np.float64), group, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s > 0, y64 / s, 0.0)
    near = _near_half_integer(v)
    bad = diff & ~near
    c = Counts(rows=u.shape[0], codes=u.size, scales=s_ref.size + z_ref.size,
               scale_mismatch=int(sm.sum() + zm.sum()), near=int((diff & near).sum()),
               bad=int(bad.sum()))
    return _finish(c, strict, "asym code", u, u_ref, bad, name)


def check_nvfp4(codes, bscales, tscale, y64, tensor_scale=None, strict=True, name=None) -> Counts:
    c_ref, sb_ref, t_ref = oracle.nvfp4(y64, tensor_scale)
    tm = np.float32(tscale).view(np.uint32) != np.float32(t_ref).view(np.uint32)
    if strict:
        assert not tm, f"tensor scale {tscale!r} != {t_ref!r}"
        assert np.array_equal(bscales, sb_ref), _first_diff(bscales, sb_ref, "E4M3 scale")
    sm = bscales != sb_ref
    c = oracle.unpack_nibbles(codes)
    diff = c != c_ref
    idx = np.nonzero(diff)                 # the window is evaluated where codes differ
    den = oracle.e4m3_decode(sb_ref)[idx[0], idx[1] // 16] * np.float64(t_ref)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.abs(np.where(den > 0, y64[idx] / den, 0.0))
    near_d = np.any(np.abs(v[:, None] - E2M1_MIDPOINTS) <= NEAR * E2M1_MIDPOINTS, axis=-1)
    # sign of a zero-magnitude code: boundary at 0
    near_d |= ((c_ref[idx] & 7) == 0) & ((c[idx] & 7) == 0) & (v <= NEAR)
    near = np.zeros_like(diff)
    near[idx] = near_d
    bad = diff & ~near
    cnt = Counts(rows=c.shape[0], codes=c.size, scales=sb_ref.size + 1,
                 scale_mismatch=int(sm.sum()) + int(tm), near=int((diff & near).sum()),
                 bad=int(bad.sum()))
    return _finish(cnt, strict, "e2m1 code", c, c_ref, bad, name)


def check_mxfp4(codes, scales, y64, strict=True, name=None) -> Counts:
    """MXFP4: E8M0 scale bytes bit-exact; codes bit-exact except within NEAR
    (relative) of an E2M1 rounding boundary, or the sign of a zero."""
    c_ref, s_ref = oracle.mxfp4(y64)
    if strict:
        assert np.array_equal(scales, s_ref), _first_diff(scales, s_ref, "E8M0 scale")
    sm = scales != s_ref
    c = oracle.unpack_nibbles(codes)
    diff = c != c_ref
    idx = np.nonzero(diff)
    X = np.ldexp(1.0, s_ref.astype(np.int64)[idx[0], idx[1] // 32] - 127)
    v = np.abs(y64[idx] / X)
    near_d = np.any(np.abs(v[:, None] - E2M1_MIDPOINTS) <= NEAR * E2M1_MIDPOINTS, axis=-1)
    near_d |= ((c_ref[idx] & 7) == 0) & ((c[idx] & 7) == 0) & (v <= NEAR)
    near = np.zeros_like(diff)
    near[idx] = near_d
    bad = diff & ~near
    cnt = Counts(rows=c.shape[0], codes=c.size, scales=s_ref.size,
                 scale_mismatch=int(sm.sum()), near=int((diff & near).sum()),
                 bad=int(bad.sum()))
    return _finish(cnt, strict, "e2m1 code", c, c_ref, bad, name)


def gpu_mxfp4(inp: wl.Inputs):
    w = inp.workload
    x, s = to_device(inp)
    codes, scales = kq.empty_mxfp4(w.tokens, w.dim)
    kq.kq_rht_quant_mxfp4(x, w.block, s, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _first_diff(a, b, what, mask=None):
    if mask is None:
        mask = a != b
    idx = np.argwhere(mask)
    if len(idx) == 0:
        return f"{what}: no difference"
    i = tuple(idx[0])
    return f"{what}: {int(mask.sum())} differences, first at {i}: got {a[i]!r} want {b[i]!r}"


# ---------------------------------------------------- whole-tensor checks
def row_chunks(tokens: int, width: int, budget: int = 1 << 23):
    """Row ranges of about `budget` elements each (bounds the oracle's
    float64 temporaries on full-size workloads)."""
    step = max(1, budget // max(width, 1))
    for r0 in range(0, tokens, step):
        yield r0, min(tokens, r0 + step)


def check_all_rows(name: str, inp: wl.Inputs, got: tuple, tensor_scale=None,
                   strict=True) -> Counts:
    """Every row of a GPU result against the oracle, in row chunks; the counts
    are recorded under `name`.  got: (codes, scales) for per-token INT4,
    (codes, scales, zeros) for asymmetric INT4, (codes, block scales, tensor
    scale) for NVFP4 (tensor_scale = the oracle's, passed in: it is global)."""
    w = inp.workload
    total = Counts()
    for r0, r1 in row_chunks(w.tokens, w.dim):
        y = oracle.rht(inp.values[r0:r1], inp.signs, w.block)
        if w.fmt == wl.INT4_SYM:
            c = check_int4_sym(got[0][r0:r1], got[1][r0:r1], y, strict, False)
        elif w.fmt == wl.INT4_ASYM:
            c = check_int4_asym(got[0][r0:r1], got[1][r0:r1], got[2][r0:r1], y, w.group, strict,
                                False)
        else:
            c = check_nvfp4(got[0][r0:r1], got[1][r0:r1], got[2], y, tensor_scale, strict,
                            False)
            if r0 > 0:
                c.scales -= 1          # the tensor scale is counted once
        total = total + c
    return record(name, total)


@functools.lru_cache(maxsize=2)
def full_inputs(key: str) -> wl.Inputs:
    """A workload's full-size inputs, kept for the next test that needs them
    (drawing the larger ones takes tens of seconds)."""
    return wl.make_inputs(wl.WORKLOADS[key])


def oracle_tensor_scale(inp: wl.Inputs) -> np.float32:
    """The oracle's dynamic NVFP4 tensor scale over every row (chunked)."""
    w = inp.workload
    g = 0.0
    for r0, r1 in row_chunks(w.tokens, w.dim):
        g = max(g, float(np.max(np.abs(oracle.rht(inp.values[r0:r1], inp.signs, w.block)))))
    return np.float32(g / (6.0 * 448.0))
