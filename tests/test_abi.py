"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/kq.h declares, and rejects bad arguments on the host before any CUDA
call (validation never dereferences the pointers, so fake aligned addresses
are enough)."""
import ctypes
import os
import re

import pytest

import hadamard_rotated_activation_b200 as kq
from hadamard_rotated_activation_b200 import build as kqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kqbuild.build()
    return kq.lib()


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "kq.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"KQ_API\s+[\w\s\*]+?\b(kq_\w+)\s*\(", src)))


def test_header_symbols_exported(L):
    names = _declared_symbols()
    assert set(names) == set(kq.C_SYMBOLS)
    for n in names:
        assert hasattr(L, n), n
        assert ctypes.cast(getattr(L, n), ctypes.c_void_p).value


def test_version_and_status_strings(L):
    assert kq.kq_version() >> 16 == 1
    for code, name in [(0, "KQ_OK"), (-1, "KQ_ERR_INVALID_ARG"), (-2, "KQ_ERR_UNSUPPORTED"),
                       (-3, "KQ_ERR_MISALIGNED"), (-4, "KQ_ERR_CUDA")]:
        assert kq.status_str(code) == name


P = 1 << 20          # a fake, 16-byte-aligned device address (never dereferenced)
Q = 2 << 20


@pytest.mark.parametrize("dim,block,want", [
    (4096, 0, 0), (4096, 128, 0), (12288, 0, 0), (12288, 128, 0), (32, 16, 0),
    (16384, 0, 0), (384, 0, 0),
    (16, 0, -2), (4095, 0, -2), (32768, 0, -2), (24576, 0, -2), (96, 0, -2),
    (4096, 8, -2), (4096, 100, -2), (4096, 8192, -2), (12288, 3072, -2),
])
def test_shape_validation(L, dim, block, want):
    # tokens = 0: a valid call is a no-op and returns KQ_OK without CUDA
    st = L.kq_rht(P, kq.KQ_BF16, 0, dim, block, None, Q, 0, None)
    assert st == want


def test_argument_errors(L):
    assert L.kq_rht(None, 1, 4, 4096, 0, None, Q, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert L.kq_rht(P, 1, -1, 4096, 0, None, Q, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert L.kq_rht(P, 7, 4, 4096, 0, None, Q, 0, None) == kq.KQ_ERR_UNSUPPORTED
    assert L.kq_rht(P, 1, 4, 4096, 0, None, None, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert L.kq_rht(P, 1, 4, 4096, 0, None, Q, 8, None) == kq.KQ_ERR_INVALID_ARG
    assert L.kq_rht(P + 2, 1, 4, 4096, 0, None, Q, 0, None) == kq.KQ_ERR_MISALIGNED
    assert L.kq_rht(P, 1, 4, 4096, 0, P + 3, Q, 0, None) == kq.KQ_ERR_MISALIGNED
    # int4: sym needs group 0 and no zeros; asym needs group 128 and zeros
    f = L.kq_rht_quant_int4
    assert f(P, 1, 0, 4096, 0, None, 0, 0, Q, Q, None, None) == kq.KQ_OK
    assert f(P, 1, 4, 4096, 0, None, 128, 0, Q, Q, None, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(P, 1, 4, 4096, 0, None, 0, 0, Q, Q, Q, None) == kq.KQ_ERR_INVALID_ARG
    assert f(P, 1, 4, 4096, 0, None, 64, 1, Q, Q, Q, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(P, 1, 4, 4096, 0, None, 128, 1, Q, Q, None, None) == kq.KQ_ERR_INVALID_ARG
    assert f(P, 1, 4, 4096, 0, None, 128, 2, Q, Q, Q, None) == kq.KQ_ERR_INVALID_ARG
    assert f(P, 1, 4, 4096, 0, None, 0, 0, Q + 4, Q, None, None) == kq.KQ_ERR_MISALIGNED
    assert f(P, 1, 4, 4096, 0, None, 0, 0, Q, Q + 2, None, None) == kq.KQ_ERR_MISALIGNED
    # nvfp4: exactly one scale mode; dynamic needs a large enough workspace
    g = L.kq_rht_quant_nvfp4
    ws = L.kq_workspace_size(4, 4096, 0)
    assert ws >= 16 + 4 * 8
    assert g(P, 1, 0, 4096, 0, None, Q, Q, Q, None, 0, kq.KQ_SCALE_STATIC, None) == kq.KQ_OK
    assert g(P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert g(P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, 6, None) == kq.KQ_ERR_INVALID_ARG
    assert g(P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, kq.KQ_SCALE_DYNAMIC, None) \
        == kq.KQ_ERR_INVALID_ARG
    assert g(P, 1, 4, 4096, 0, None, Q, Q, Q, P, ws - 1, kq.KQ_SCALE_DYNAMIC, None) \
        == kq.KQ_ERR_INVALID_ARG
    assert g(P, 1, 4, 4096, 0, None, Q, Q, Q, P + 8, ws, kq.KQ_SCALE_DYNAMIC, None) \
        == kq.KQ_ERR_MISALIGNED
    assert g(P, 1, 0, 4096, 0, None, Q, Q, Q, P, ws, kq.KQ_SCALE_DYNAMIC, None) == kq.KQ_OK
    # dequant
    d = L.kq_dequant
    assert d(4, Q, Q, None, None, 4, 4096, 0, P, None) == kq.KQ_ERR_INVALID_ARG
    assert d(2, Q, Q, None, None, 4, 4096, 0, P, None) == kq.KQ_ERR_INVALID_ARG
    assert d(1, Q, Q, None, None, 4, 4096, 128, P, None) == kq.KQ_ERR_INVALID_ARG
    assert d(1, Q, Q, Q, None, 4, 4096, 64, P, None) == kq.KQ_ERR_UNSUPPORTED
    assert d(0, Q, Q, None, None, 4, 4100, 0, P, None) == kq.KQ_ERR_UNSUPPORTED
    assert d(0, Q, Q, None, None, 0, 4096, 0, P, None) == kq.KQ_OK
    # tokens == 0: data pointers may be NULL
    assert L.kq_rht(None, 1, 0, 4096, 0, None, None, 0, None) == kq.KQ_OK
    assert d(2, None, None, None, None, 0, 4096, 0, None, None) == kq.KQ_OK
    assert L.kq_workspace_size(4, 4095, 0) == 0
    assert L.kq_device_errors(None) == kq.KQ_ERR_INVALID_ARG
    assert L.kq_diag_wait_timeout(0, None) == kq.KQ_ERR_INVALID_ARG
    assert L.kq_diag_wait_timeout(5_000_000_000, None) == kq.KQ_ERR_INVALID_ARG
    # KV writer: bf16, block 128, group 128; all buffers present and aligned
    v = L.kq_rht_quant_int4_kv
    assert v(P, 1, 0, 4096, 128, None, 128, Q, 16, Q, Q, Q, None) == kq.KQ_OK
    assert v(P, 1, 4, 4096, 128, None, 128, Q, -1, Q, Q, Q, None) == kq.KQ_ERR_INVALID_ARG
    assert v(P, 1, 4, 4096, 128, None, 128, None, 16, Q, Q, Q, None) == kq.KQ_ERR_INVALID_ARG
    assert v(P, 0, 4, 4096, 128, None, 128, Q, 16, Q, Q, Q, None) == kq.KQ_ERR_UNSUPPORTED
    assert v(P, 1, 4, 4096, 0, None, 128, Q, 16, Q, Q, Q, None) == kq.KQ_ERR_UNSUPPORTED
    assert v(P, 1, 4, 4096, 128, None, 64, Q, 16, Q, Q, Q, None) == kq.KQ_ERR_UNSUPPORTED
    assert v(P, 1, 4, 4096, 128, None, 128, Q + 4, 16, Q, Q, Q, None) == kq.KQ_ERR_MISALIGNED
    assert v(P, 1, 4, 4096, 128, P + 8, 128, Q, 16, Q, Q, Q, None) == kq.KQ_ERR_MISALIGNED
    assert v(P, 1, 4, 4096, 128, None, 128, Q, 16, Q + 8, Q, Q, None) == kq.KQ_ERR_MISALIGNED
    # mxfp4: the rotation's checks, codes 16-byte aligned
    m = L.kq_rht_quant_mxfp4
    assert m(P, 1, 0, 4096, 0, None, Q, Q, None) == kq.KQ_OK
    assert m(P, 1, 4, 4096, 0, None, None, Q, None) == kq.KQ_ERR_INVALID_ARG
    assert m(P, 1, 4, 4096, 0, None, Q, None, None) == kq.KQ_ERR_INVALID_ARG
    assert m(P, 1, 4, 4096, 0, None, Q + 8, Q, None) == kq.KQ_ERR_MISALIGNED
    assert m(P, 1, 4, 4095, 0, None, Q, Q, None) == kq.KQ_ERR_UNSUPPORTED
    assert m(P, 3, 4, 4096, 0, None, Q, Q, None) == kq.KQ_ERR_UNSUPPORTED
    assert d(3, Q, Q + 1, None, None, 0, 4096, 0, P, None) == kq.KQ_OK
    # dequant + inverse rotation: the rotation's shape checks, then dequant's
    r = L.kq_dequant_rht_inverse
    assert r(2, Q, Q, None, P, 4, 4096, 0, 0, None, P, 2, None) == kq.KQ_ERR_UNSUPPORTED
    assert r(2, Q, Q, None, P, 0, 4096, 0, 0, None, P, 0, None) == kq.KQ_OK
    assert r(2, None, None, None, None, 0, 4096, 0, 0, None, None, 0, None) == kq.KQ_OK
    assert r(2, Q, Q, None, P, -1, 4096, 0, 0, None, P, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert r(2, Q, Q, None, P, 4, 4095, 0, 0, None, P, 0, None) == kq.KQ_ERR_UNSUPPORTED
    assert r(2, Q, Q, None, P, 4, 4096, 100, 0, None, P, 0, None) == kq.KQ_ERR_UNSUPPORTED
    assert r(2, Q, Q, None, None, 4, 4096, 0, 0, None, P, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert r(2, Q, Q, None, P, 4, 4096, 0, 0, None, None, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert r(2, Q, Q, None, P, 4, 4096, 0, 0, P + 4, P, 0, None) == kq.KQ_ERR_MISALIGNED
    assert r(2, Q, Q, None, P, 4, 4096, 0, 0, None, P + 4, 0, None) == kq.KQ_ERR_MISALIGNED
    assert r(2, Q + 8, Q, None, P, 4, 4096, 0, 0, None, P, 0, None) == kq.KQ_ERR_MISALIGNED
    assert r(1, Q, Q, None, None, 4, 4096, 0, 128, None, P, 0, None) == kq.KQ_ERR_INVALID_ARG
    assert r(1, Q, Q, Q, None, 4, 4096, 0, 64, None, P, 0, None) == kq.KQ_ERR_UNSUPPORTED
    assert r(0, Q, Q + 2, None, None, 4, 4096, 0, 0, None, P, 0, None) == kq.KQ_ERR_MISALIGNED
    assert r(5, Q, Q, None, None, 4, 4096, 0, 0, None, P, 0, None) == kq.KQ_ERR_INVALID_ARG
    t = L.kq_diag_tc_steps
    assert t(None, P, P, P, P, None) == kq.KQ_ERR_INVALID_ARG
    assert t(P + 1, P, P, P, P, None) == kq.KQ_ERR_MISALIGNED
    assert t(P, P, P + 2, P, P, None) == kq.KQ_ERR_MISALIGNED


def test_python_binding_rejects_host_tensors(L):
    import torch
    x = torch.zeros(2, 64)
    with pytest.raises(ValueError):
        kq.kq_rht(x, 0, None, torch.zeros(2, 64))


# cudaErrorLaunchOutOfResources, a launch failure a real GPU can report
_LAUNCH_ERR = 701


def test_launch_failure_reaches_the_caller(L):
    """A simulated launch failure (armed by kq_diag_fail_next_launch, so that
    nothing is launched and no GPU is needed) comes back from each entry point
    as KQ_ERR_CUDA with the CUDA error in kq_last_cuda_error()."""
    ws = L.kq_workspace_size(4, 4096, 0)
    calls = {
        "kq_rht": lambda: L.kq_rht(P, kq.KQ_BF16, 4, 4096, 0, None, Q, 0, None),
        "kq_rht inverse": lambda: L.kq_rht(P, kq.KQ_F32, 4, 12288, 0, None, Q, kq.KQ_INVERSE,
                                           None),
        "kq_rht_quant_int4 sym": lambda: L.kq_rht_quant_int4(P, 1, 4, 12288, 0, None, 0, 0, Q,
                                                            Q, None, None),
        "kq_rht_quant_int4 asym": lambda: L.kq_rht_quant_int4(P, 1, 4, 4096, 128, None, 128, 1,
                                                             Q, Q, Q, None),
        "kq_rht_quant_nvfp4 static": lambda: L.kq_rht_quant_nvfp4(
            P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, kq.KQ_SCALE_STATIC, None),
        "kq_rht_quant_nvfp4 dynamic": lambda: L.kq_rht_quant_nvfp4(
            P, 1, 4, 4096, 128, None, Q, Q, Q, P, ws, kq.KQ_SCALE_DYNAMIC, None),
        "kq_rht_quant_mxfp4": lambda: L.kq_rht_quant_mxfp4(P, 1, 4, 4096, 0, None, Q, Q, None),
        "kq_dequant": lambda: L.kq_dequant(kq.KQ_FMT_INT4_SYM, P, Q, None, None, 4, 4096, 0, Q,
                                           None),
        "kq_dequant_rht_inverse": lambda: L.kq_dequant_rht_inverse(
            kq.KQ_FMT_NVFP4, P, Q, None, Q, 4, 4096, 0, 0, None, Q, kq.KQ_F32, None),
        "kq_rht_quant_int4_kv": lambda: L.kq_rht_quant_int4_kv(P, 1, 4, 4096, 128, None, 128, P,
                                                               8, Q, Q, Q, None),
        "kq_diag_wait_timeout": lambda: L.kq_diag_wait_timeout(1000, None),
    }
    try:
        for name, call in calls.items():
            L.kq_diag_fail_next_launch(_LAUNCH_ERR)
            assert call() == kq.KQ_ERR_CUDA, name
            assert L.kq_last_cuda_error() == _LAUNCH_ERR, name
        # a call its checks reject, or a no-op call, does not take the failure
        L.kq_diag_fail_next_launch(_LAUNCH_ERR + 1)
        assert L.kq_rht(P + 2, 1, 4, 4096, 0, None, Q, 0, None) == kq.KQ_ERR_MISALIGNED
        assert L.kq_rht(P, 1, 0, 4096, 0, None, Q, 0, None) == kq.KQ_OK
        assert L.kq_rht(P, 1, 4, 4096, 0, None, Q, 0, None) == kq.KQ_ERR_CUDA
        assert L.kq_last_cuda_error() == _LAUNCH_ERR + 1
        # the Python binding raises with the CUDA error in the message
        L.kq_diag_fail_next_launch(_LAUNCH_ERR)
        with pytest.raises(kq.KQError, match="701"):
            kq._check(L.kq_rht(P, 1, 4, 4096, 0, None, Q, 0, None), "kq_rht")
    finally:
        L.kq_diag_fail_next_launch(0)


def test_gemm_and_scale_layout_validation(L):
    """Host-side checks of kq_gemm_nvfp4 and of the KQ_SCALES_MMA flag."""
    g = L.kq_gemm_nvfp4
    ok = (P, Q, P, Q, P, Q)
    assert g(*ok, 0, 4096, 4096, Q, kq.KQ_F32, None) == kq.KQ_OK          # m = 0: no-op
    assert g(*ok, -1, 4096, 4096, Q, kq.KQ_F32, None) == kq.KQ_ERR_INVALID_ARG
    assert g(*ok, 4, 0, 4096, Q, kq.KQ_F32, None) == kq.KQ_ERR_INVALID_ARG
    assert g(*ok, 4, 4096, 4096, Q, 7, None) == kq.KQ_ERR_UNSUPPORTED
    assert g(*ok, 4, 4000, 4096, Q, kq.KQ_F32, None) == kq.KQ_ERR_UNSUPPORTED   # n % 128
    assert g(*ok, 4, 4096, 4000, Q, kq.KQ_F32, None) == kq.KQ_ERR_UNSUPPORTED   # k % 256
    assert g(None, Q, P, Q, P, Q, 4, 4096, 4096, Q, kq.KQ_F32, None) == kq.KQ_ERR_INVALID_ARG
    assert g(P + 8, Q, P, Q, P, Q, 4, 4096, 4096, Q, kq.KQ_F32, None) == kq.KQ_ERR_MISALIGNED
    assert g(*ok, 4, 4096, 4096, Q + 8, kq.KQ_BF16, None) == kq.KQ_ERR_MISALIGNED
    f = L.kq_rht_quant_nvfp4
    mma = kq.KQ_SCALE_STATIC | kq.KQ_SCALES_MMA
    assert f(P, 1, 0, 4096, 0, None, Q, Q, Q, None, 0, mma, None) == kq.KQ_OK
    assert f(P, 1, 4, 32, 0, None, Q, Q, Q, None, 0, mma, None) == kq.KQ_ERR_UNSUPPORTED
    assert f(P, 1, 4, 4096, 0, None, Q, Q + 4, Q, None, 0, mma, None) == kq.KQ_ERR_MISALIGNED
    assert f(P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, mma | 16, None) == kq.KQ_ERR_INVALID_ARG
    try:
        L.kq_diag_fail_next_launch(_LAUNCH_ERR)
        assert g(*ok, 4, 4096, 4096, Q, kq.KQ_F32, None) == kq.KQ_ERR_CUDA
        assert L.kq_last_cuda_error() == _LAUNCH_ERR
        L.kq_diag_fail_next_launch(_LAUNCH_ERR)
        assert f(P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, mma, None) == kq.KQ_ERR_CUDA
    finally:
        L.kq_diag_fail_next_launch(0)


def test_dynamic_phase_flags_validation(L):
    f = L.kq_rht_quant_nvfp4
    ws = L.kq_workspace_size(4, 4096, 0)
    static = kq.KQ_SCALE_STATIC
    dyn = kq.KQ_SCALE_DYNAMIC
    for ph in (kq.KQ_DYN_STATS, kq.KQ_DYN_EXACT, kq.KQ_DYN_QUANT):
        assert f(P, 1, 4, 4096, 0, None, Q, Q, Q, None, 0, static | ph, None) == \
            kq.KQ_ERR_INVALID_ARG
        assert f(P, 1, 0, 4096, 0, None, Q, Q, Q, P, ws, dyn | ph, None) == kq.KQ_OK
    assert f(P, 1, 4, 4096, 0, None, Q, Q, Q, P, ws, dyn | 128, None) == kq.KQ_ERR_INVALID_ARG
    try:
        L.kq_diag_fail_next_launch(_LAUNCH_ERR)
        assert f(P, 1, 4, 4096, 0, None, Q, Q, Q, P, ws, dyn | kq.KQ_DYN_EXACT, None) == \
            kq.KQ_ERR_CUDA
    finally:
        L.kq_diag_fail_next_launch(0)
