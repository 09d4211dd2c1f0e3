"""The allocation-free dynamic NVFP4 entry point gives exactly what the
workspace-taking entry point gives.

Callers such as a framework plugin that is handed no device workspace, or a
serving loop that may not call cudaMalloc on its hot path, use
kq_rht_quant_nvfp4_dynamic_noalloc; its workspace is a fixed array inside the
library.  This file is collected last so that a failure here leaves every other
test already run.  It must pass on its own in a fresh process too.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import hadamard_rotated_activation_b200 as kq
from hadamard_rotated_activation_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _device_input(key, tokens):
    inp = wl.make_inputs(wl.WORKLOADS[key], tokens=tokens)
    x = torch.from_numpy(inp.stored.view(np.int16)).cuda().view(torch.bfloat16)
    s = torch.from_numpy(inp.signs).cuda()
    return x, s


@pytest.mark.parametrize("key,tokens", [("c4", 301), ("c2", 77)])
def test_noalloc_matches_workspace_entry_point(key, tokens):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = kq.lib()
    w = wl.WORKLOADS[key]
    x, s = _device_input(key, tokens)
    stream = torch.cuda.current_stream().cuda_stream

    # reference: the existing entry point with a caller-allocated workspace
    c_ref, b_ref, t_ref, ws = kq.empty_nvfp4(tokens, w.dim, w.block)
    st = L.kq_rht_quant_nvfp4(x.data_ptr(), kq.KQ_BF16, tokens, w.dim, w.block, s.data_ptr(),
                              c_ref.data_ptr(), b_ref.data_ptr(), t_ref.data_ptr(),
                              ws.data_ptr(), ws.numel(), kq.KQ_SCALE_DYNAMIC, stream)
    assert st == kq.KQ_OK, kq.status_str(st)
    torch.cuda.synchronize()

    # two calls in a row through the C ABI: the shared scratch keeps the
    # previous call's contents, which must not leak into the next result
    for _ in range(2):
        c = torch.full_like(c_ref, 0xAB)
        b = torch.full_like(b_ref, 0xCD)
        t = torch.full_like(t_ref, -1.0)
        st = L.kq_rht_quant_nvfp4_dynamic_noalloc(
            x.data_ptr(), kq.KQ_BF16, tokens, w.dim, w.block, s.data_ptr(),
            c.data_ptr(), b.data_ptr(), t.data_ptr(), stream)
        assert st == kq.KQ_OK, kq.status_str(st)
        torch.cuda.synchronize()
        # bit-exact, the tolerance the parity tests use for codes and scales
        assert torch.equal(c, c_ref)
        assert torch.equal(b, b_ref)
        assert torch.equal(t.view(torch.int32), t_ref.view(torch.int32))


def test_noalloc_rejects_too_many_tokens():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = kq.lib()
    big = kq.KQ_NOALLOC_MAX_TOKENS + 1
    P = 1 << 20
    st = L.kq_rht_quant_nvfp4_dynamic_noalloc(P, kq.KQ_BF16, big, 4096, 0, None, P, P, P, None)
    assert st == kq.KQ_ERR_UNSUPPORTED


def _call_pair(L, x, s, tokens, dim, block, stream):
    """(reference with a fresh workspace, allocation-free) outputs of one input."""
    c_ref, b_ref, t_ref, ws = kq.empty_nvfp4(tokens, dim, block)
    st = L.kq_rht_quant_nvfp4(x.data_ptr(), kq.KQ_BF16, tokens, dim, block, s.data_ptr(),
                              c_ref.data_ptr(), b_ref.data_ptr(), t_ref.data_ptr(),
                              ws.data_ptr(), ws.numel(), kq.KQ_SCALE_DYNAMIC, stream)
    assert st == kq.KQ_OK, kq.status_str(st)
    c = torch.full_like(c_ref, 0xAB)
    b = torch.full_like(b_ref, 0xCD)
    t = torch.full_like(t_ref, -1.0)
    st = L.kq_rht_quant_nvfp4_dynamic_noalloc(x.data_ptr(), kq.KQ_BF16, tokens, dim, block,
                                              s.data_ptr(), c.data_ptr(), b.data_ptr(),
                                              t.data_ptr(), stream)
    assert st == kq.KQ_OK, kq.status_str(st)
    torch.cuda.synchronize()
    return (c_ref, b_ref, t_ref), (c, b, t)


@pytest.mark.parametrize("dim", [2048, 12288])
def test_noalloc_dirty_scratch_header_only_paths(dim):
    """Paths that clear only the scratch's header (the warp-per-row kernel for
    2048-wide rows, the row-per-CTA kernel for 12288) rely on their statistics
    pass rewriting every row entry before the global step reads it: a larger
    call leaves the scratch dirty, then a smaller call must still match."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = kq.lib()
    stream = torch.cuda.current_stream().cuda_stream
    big, small = 600, 37
    w = wl.Workload("c4", big, dim, wl.BF16, 0, True, wl.NVFP4, seed=dim)
    inp = wl.make_inputs(w)
    x = torch.from_numpy(inp.stored.view(np.int16)).cuda().view(torch.bfloat16)
    s = torch.from_numpy(inp.signs).cuda()
    # the small call's rows get the largest values, so stale entries of the
    # big call (smaller maxima) cannot hide a missed rewrite
    x_small = (x[:small].float() * 4).to(torch.bfloat16).contiguous()
    for xx, n in ((x, big), (x_small, small)):
        ref, got = _call_pair(L, xx, s, n, dim, 0, stream)
        for a, b in zip(ref, got):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
