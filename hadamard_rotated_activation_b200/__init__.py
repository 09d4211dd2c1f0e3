"""Fused randomized Hadamard rotation + 4-bit quantization of activations (B200).

Thin ctypes binding over the C ABI in include/kq.h (libkq.so, built in-tree by
`python -m hadamard_rotated_activation_b200.build`).  Functions carry the C
names and only marshal arguments: torch CUDA tensors become device pointers and
the current torch stream becomes the kq stream.  Every step of the path runs in
the library's CUDA kernels; there is no other implementation here, and a
missing library is an error.

PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkq.so")

KQ_OK = 0
KQ_ERR_INVALID_ARG = -1
KQ_ERR_UNSUPPORTED = -2
KQ_ERR_MISALIGNED = -3
KQ_ERR_CUDA = -4

KQ_F32 = 0
KQ_BF16 = 1

KQ_INVERSE = 1
KQ_SCALE_STATIC = 2
KQ_SCALE_DYNAMIC = 4
KQ_SCALES_MMA = 8
KQ_DYN_STATS = 16
KQ_DYN_EXACT = 32
KQ_DYN_QUANT = 64

KQ_FMT_INT4_SYM = 0
KQ_FMT_INT4_ASYM = 1
KQ_FMT_NVFP4 = 2
KQ_FMT_MXFP4 = 3

C_SYMBOLS = (
    "kq_rht", "kq_rht_quant_int4", "kq_rht_quant_nvfp4", "kq_dequant",
    "kq_dequant_rht_inverse", "kq_rht_quant_mxfp4", "kq_rht_quant_int4_kv",
    "kq_device_errors", "kq_diag_wait_timeout",
    "kq_workspace_size", "kq_status_str", "kq_last_cuda_error", "kq_version",
    "kq_rht_quant_nvfp4_dynamic_noalloc", "kq_diag_tc_steps", "kq_diag_fail_next_launch",
    "kq_gemm_nvfp4", "kq_diag_tc_steps_f16",
)

# Fixed device scratch of kq_rht_quant_nvfp4_dynamic_noalloc (see include/kq.h).
KQ_NOALLOC_SCRATCH_BYTES = 1 << 20
KQ_NOALLOC_MAX_TOKENS = (KQ_NOALLOC_SCRATCH_BYTES - 16) // 8

_lib = None


class KQError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {status_str(status)} ({status})"
        if status == KQ_ERR_CUDA:
            msg += f", cuda error {lib().kq_last_cuda_error()}"
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libkq.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m hadamard_rotated_activation_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.kq_rht.argtypes = [vp, i32, i64, i32, i32, vp, vp, i32, vp]
    L.kq_rht.restype = i32
    L.kq_rht_quant_int4.argtypes = [vp, i32, i64, i32, i32, vp, i32, i32, vp, vp, vp, vp]
    L.kq_rht_quant_int4.restype = i32
    L.kq_rht_quant_nvfp4.argtypes = [vp, i32, i64, i32, i32, vp, vp, vp, vp, vp, sz, i32, vp]
    L.kq_rht_quant_nvfp4.restype = i32
    L.kq_dequant.argtypes = [i32, vp, vp, vp, vp, i64, i32, i32, vp, vp]
    L.kq_dequant.restype = i32
    L.kq_rht_quant_mxfp4.argtypes = [vp, i32, i64, i32, i32, vp, vp, vp, vp]
    L.kq_rht_quant_mxfp4.restype = i32
    L.kq_rht_quant_int4_kv.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp, i64, vp, vp, vp, vp]
    L.kq_rht_quant_int4_kv.restype = i32
    L.kq_device_errors.argtypes = [vp]
    L.kq_device_errors.restype = i32
    L.kq_diag_wait_timeout.argtypes = [ctypes.c_longlong, vp]
    L.kq_diag_wait_timeout.restype = i32
    L.kq_dequant_rht_inverse.argtypes = [i32, vp, vp, vp, vp, i64, i32, i32, i32, vp, vp, i32,
                                         vp]
    L.kq_dequant_rht_inverse.restype = i32
    L.kq_rht_quant_nvfp4_dynamic_noalloc.argtypes = [vp, i32, i64, i32, i32, vp, vp, vp,
                                                     vp, vp]
    L.kq_rht_quant_nvfp4_dynamic_noalloc.restype = i32
    L.kq_workspace_size.argtypes = [i64, i32, i32]
    L.kq_workspace_size.restype = sz
    L.kq_status_str.argtypes = [i32]
    L.kq_status_str.restype = ctypes.c_char_p
    L.kq_last_cuda_error.argtypes = []
    L.kq_last_cuda_error.restype = i32
    L.kq_version.argtypes = []
    L.kq_version.restype = i32
    L.kq_diag_tc_steps.argtypes = [vp, vp, vp, vp, vp, vp]
    L.kq_diag_tc_steps.restype = i32
    L.kq_diag_fail_next_launch.argtypes = [i32]
    L.kq_diag_fail_next_launch.restype = None
    L.kq_diag_tc_steps_f16.argtypes = [vp, vp, vp, vp, vp, vp]
    L.kq_diag_tc_steps_f16.restype = i32
    L.kq_gemm_nvfp4.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, i32, vp]
    L.kq_gemm_nvfp4.restype = i32
    _lib = L
    return L


def status_str(status: int) -> str:
    return lib().kq_status_str(int(status)).decode()


# ------------------------------------------------------------ marshalling
def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("kq functions take CUDA tensors (device pointers)")
    if not t.is_contiguous():
        raise ValueError("kq functions take contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(x) -> int:
    import torch
    if x.dtype == torch.bfloat16:
        return KQ_BF16
    if x.dtype == torch.float32:
        return KQ_F32
    raise ValueError(f"unsupported input dtype {x.dtype}")


def _check(status: int, where: str) -> None:
    if status != KQ_OK:
        raise KQError(status, where)


# -------------------------------------------------------------- C names
def kq_rht(x, block: int, signs, out, inverse: bool = False, stream=None) -> None:
    """Rotation only (fp32 out): forward y = x D H^T / sqrt(b), or the inverse."""
    t, n = x.shape
    _check(lib().kq_rht(_ptr(x), _dtype_code(x), t, n, block, _ptr(signs), _ptr(out),
                        KQ_INVERSE if inverse else 0, _stream(stream)), "kq_rht")


def kq_rht_quant_int4(x, block: int, signs, group: int, asym: bool, codes, scales,
                      zeros=None, stream=None) -> None:
    """Rotation + INT4: symmetric per token (group 0, fp32 scales) or
    asymmetric per group of 128 (fp16 scales and zero-points)."""
    t, n = x.shape
    _check(lib().kq_rht_quant_int4(_ptr(x), _dtype_code(x), t, n, block, _ptr(signs),
                                   group, 1 if asym else 0, _ptr(codes), _ptr(scales),
                                   _ptr(zeros), _stream(stream)), "kq_rht_quant_int4")


def kq_rht_quant_nvfp4(x, block: int, signs, codes, block_scales, tensor_scale,
                       workspace=None, dynamic: bool = True, stream=None,
                       mma_layout: bool = False, phases: int = 0) -> None:
    """Rotation + NVFP4 (E2M1 codes, E4M3 scale per 16, fp32 tensor scale).
    dynamic=True computes and writes the tensor scale (needs `workspace` of
    kq_workspace_size bytes); dynamic=False reads it.  mma_layout=True writes
    the block scales in the tensor-core layout kq_gemm_nvfp4 reads (a buffer
    of sf_mma_bytes(tokens, dim) bytes)."""
    t, n = x.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    flags = ((KQ_SCALE_DYNAMIC if dynamic else KQ_SCALE_STATIC) |
             (KQ_SCALES_MMA if mma_layout else 0) | phases)
    _check(lib().kq_rht_quant_nvfp4(_ptr(x), _dtype_code(x), t, n, block, _ptr(signs),
                                    _ptr(codes), _ptr(block_scales), _ptr(tensor_scale),
                                    _ptr(workspace), ws_bytes, flags, _stream(stream)),
           "kq_rht_quant_nvfp4")


def kq_rht_quant_int4_kv(x, signs, slot_mapping, codes_cache, scales_cache, zeros_cache,
                         stream=None) -> None:
    """Rotation (per-head H_128) + asymmetric INT4 g128 into KV-cache rows:
    token t lands in row slot_mapping[t] (int64; negative = skip)."""
    t, n = x.shape
    _check(lib().kq_rht_quant_int4_kv(_ptr(x), _dtype_code(x), t, n, 128, _ptr(signs), 128,
                                      _ptr(slot_mapping), codes_cache.shape[0],
                                      _ptr(codes_cache), _ptr(scales_cache), _ptr(zeros_cache),
                                      _stream(stream)),
           "kq_rht_quant_int4_kv")


def kq_rht_quant_mxfp4(x, block: int, signs, codes, scales, stream=None) -> None:
    """Rotation + MXFP4 (E2M1 codes, one E8M0 scale byte per 32 elements)."""
    t, n = x.shape
    _check(lib().kq_rht_quant_mxfp4(_ptr(x), _dtype_code(x), t, n, block, _ptr(signs),
                                    _ptr(codes), _ptr(scales), _stream(stream)),
           "kq_rht_quant_mxfp4")


def kq_rht_quant_nvfp4_dynamic_noalloc(x, block: int, signs, codes, block_scales,
                                       tensor_scale, stream=None) -> None:
    """Dynamic-scale NVFP4 for callers that cannot allocate device memory: the
    workspace is the library's own fixed device array (at most
    KQ_NOALLOC_MAX_TOKENS rows).  Calls that overlap on the GPU race."""
    t, n = x.shape
    _check(lib().kq_rht_quant_nvfp4_dynamic_noalloc(
        _ptr(x), _dtype_code(x), t, n, block, _ptr(signs), _ptr(codes), _ptr(block_scales),
        _ptr(tensor_scale), _stream(stream)), "kq_rht_quant_nvfp4_dynamic_noalloc")


def sharded_dynamic_protocol(run_phase, lower, gmax, all_reduce_max, empty: bool) -> None:
    """The order of a sharded dynamic NVFP4 call on one rank: phase 1, MAX
    over the ranks of the lower bound (`lower`, the workspace's bytes 0-3 as
    int32), phase 2, MAX of the exact maximum (`gmax`, bytes 8-15 as int64),
    phase 3.  Every rank takes both collectives, a rank with no rows too (it
    contributes zeros).  run_phase(flag) runs one phase of the library."""
    if empty:
        lower.zero_()
        gmax.zero_()
    else:
        run_phase(KQ_DYN_STATS)
    all_reduce_max(lower)
    if not empty:
        run_phase(KQ_DYN_EXACT)
    all_reduce_max(gmax)
    if not empty:
        run_phase(KQ_DYN_QUANT)


def nvfp4_dynamic_sharded(x, block: int, signs, codes, block_scales, tensor_scale, workspace,
                          all_reduce_max, stream=None, mma_layout: bool = False) -> None:
    """Dynamic NVFP4 of a tensor whose rows are split over ranks: every rank
    gets the tensor scale of the whole tensor (the single-call result).
    all_reduce_max(t) reduces a one-element int32 or int64 device tensor in
    place with MAX over the ranks (torch.distributed.all_reduce with
    ReduceOp.MAX, say).  See kq_rht_quant_nvfp4 in include/kq.h."""
    torch = _torch()
    ws8 = workspace.view(-1)

    def run(flag):
        kq_rht_quant_nvfp4(x, block, signs, codes, block_scales, tensor_scale, workspace, True,
                           stream=stream, mma_layout=mma_layout, phases=flag)
    sharded_dynamic_protocol(run, ws8[0:4].view(torch.int32), ws8[8:16].view(torch.int64),
                             all_reduce_max, x.shape[0] == 0)


def _torch():
    import torch
    return torch


def kq_gemm_nvfp4(a_codes, a_scales, a_tensor_scale, b_codes, b_scales, b_tensor_scale, c,
                  stream=None) -> None:
    """C = ta tb A_q B_q^T on the block-scaled tensor cores: A [m, k/2] and B
    [n, k/2] packed E2M1 codes with block scales in the tensor-core layout
    (kq_rht_quant_nvfp4(..., mma_layout=True)); C [m, n] fp32 or bf16."""
    m, kb = a_codes.shape
    n = b_codes.shape[0]
    _check(lib().kq_gemm_nvfp4(_ptr(a_codes), _ptr(a_scales), _ptr(a_tensor_scale),
                               _ptr(b_codes), _ptr(b_scales), _ptr(b_tensor_scale), m, n,
                               2 * kb, _ptr(c), _dtype_code(c), _stream(stream)),
           "kq_gemm_nvfp4")


def kq_dequant(fmt: int, codes, scales, zeros, tensor_scale, tokens: int, dim: int,
               group: int, out, stream=None) -> None:
    """Codes and scales back to fp32 (exact product, one rounding)."""
    _check(lib().kq_dequant(fmt, _ptr(codes), _ptr(scales), _ptr(zeros),
                            _ptr(tensor_scale), tokens, dim, group, _ptr(out),
                            _stream(stream)), "kq_dequant")


def kq_dequant_rht_inverse(fmt: int, codes, scales, zeros, tensor_scale, tokens: int,
                           dim: int, block: int, group: int, signs, out, stream=None) -> None:
    """Dequantize and undo the rotation in one call; `out` is fp32 or bf16."""
    _check(lib().kq_dequant_rht_inverse(fmt, _ptr(codes), _ptr(scales), _ptr(zeros),
                                        _ptr(tensor_scale), tokens, dim, block, group,
                                        _ptr(signs), _ptr(out), _dtype_code(out),
                                        _stream(stream)),
           "kq_dequant_rht_inverse")


def kq_diag_tc_steps(a, b, d1, d2, status, stream=None, fp16=False) -> None:
    """Two tensor-core accumulation steps on caller data (diagnostic; see
    include/kq.h): a bf16 (fp16 with fp16=True) [128, 32], b [32, 128], d1/d2
    fp32 [128, 128], status one int32 (0 = the waits completed)."""
    fn = lib().kq_diag_tc_steps_f16 if fp16 else lib().kq_diag_tc_steps
    _check(fn(_ptr(a), _ptr(b), _ptr(d1), _ptr(d2), _ptr(status), _stream(stream)),
           "kq_diag_tc_steps")


def kq_device_errors():
    """The six error words of the tensor-core kernel families (read and
    cleared): 4096-wide, 12288-wide, block-128 GEMM, fused inverse,
    diagnostic, NVFP4 GEMM.  All zero: no bounded wait ran out since the last
    call."""
    buf = (ctypes.c_uint * 6)()
    _check(lib().kq_device_errors(buf), "kq_device_errors")
    return list(buf)


def kq_diag_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Diagnostic: a wait that nothing satisfies, bounded by limit_cycles."""
    _check(lib().kq_diag_wait_timeout(int(limit_cycles), _stream(stream)),
           "kq_diag_wait_timeout")


def kq_workspace_size(tokens: int, dim: int, block: int) -> int:
    return int(lib().kq_workspace_size(tokens, dim, block))


def kq_version() -> int:
    return int(lib().kq_version())


# ------------------------------------------------- output allocation helpers
def empty_int4_sym(tokens: int, dim: int, device="cuda"):
    import torch
    return (torch.empty((tokens, dim // 2), dtype=torch.uint8, device=device),
            torch.empty((tokens,), dtype=torch.float32, device=device))


def empty_int4_asym(tokens: int, dim: int, group: int = 128, device="cuda"):
    import torch
    g = dim // group
    return (torch.empty((tokens, dim // 2), dtype=torch.uint8, device=device),
            torch.empty((tokens, g), dtype=torch.float16, device=device),
            torch.empty((tokens, g), dtype=torch.float16, device=device))


def empty_mxfp4(tokens: int, dim: int, device="cuda"):
    """(codes, scales) for kq_rht_quant_mxfp4."""
    import torch
    return (torch.empty((tokens, dim // 2), dtype=torch.uint8, device=device),
            torch.empty((tokens, dim // 32), dtype=torch.uint8, device=device))


def sf_mma_bytes(rows: int, dim: int) -> int:
    """Bytes of NVFP4 block scales in the tensor-core layout: rows padded to a
    multiple of 128, dim / 16 scales a row (dim % 64 == 0)."""
    return -(-rows // 128) * 128 * (dim // 16)


def empty_nvfp4(tokens: int, dim: int, block: int = 0, device="cuda", mma_layout=False):
    """(codes, block_scales, tensor_scale, workspace) for kq_rht_quant_nvfp4;
    with mma_layout the block scales are a flat buffer of sf_mma_bytes."""
    import torch
    ws = kq_workspace_size(tokens, dim, block)
    scales = (torch.zeros((sf_mma_bytes(tokens, dim),), dtype=torch.uint8, device=device)
              if mma_layout else
              torch.empty((tokens, dim // 16), dtype=torch.uint8, device=device))
    return (torch.empty((tokens, dim // 2), dtype=torch.uint8, device=device),
            scales,
            torch.empty((1,), dtype=torch.float32, device=device),
            torch.empty((max(ws, 16),), dtype=torch.uint8, device=device))
