"""Failure reports of the tensor-core kernels on a GPU, without a fault: the
words stay clear after ordinary calls, and a wait that nothing satisfies
(the diagnostic entry point, bounded to about a millisecond) sets its word,
which the read then clears."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import hadamard_rotated_activation_b200 as kq
from hadamard_rotated_activation_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


def test_words_clear_after_ordinary_calls():
    kq.kq_device_errors()                          # start from a clear state
    w = wl.WORKLOADS["c4"].with_tokens(128)
    inp = wl.make_inputs(w)
    x = torch.from_numpy(inp.stored.view(np.int16)).cuda().view(torch.bfloat16)
    s = torch.from_numpy(inp.signs).cuda()
    c, bs, ts, ws = kq.empty_nvfp4(w.tokens, w.dim, 0)
    kq.kq_rht_quant_nvfp4(x, 0, s, c, bs, ts, ws, dynamic=True)
    out = torch.empty((w.tokens, w.dim), dtype=torch.float32, device="cuda")
    kq.kq_rht(x, 0, s, out)
    cm, bm, tm, _ = kq.empty_nvfp4(w.tokens, w.dim, 0, mma_layout=True)
    tm.copy_(ts)
    kq.kq_rht_quant_nvfp4(x, 0, s, cm, bm, tm, None, dynamic=False, mma_layout=True)
    g = torch.empty((w.tokens, 128), dtype=torch.float32, device="cuda")
    kq.kq_gemm_nvfp4(cm, bm, tm, cm, bm, tm, g)
    torch.cuda.synchronize()
    assert kq.kq_device_errors() == [0, 0, 0, 0, 0, 0]


def test_bounded_wait_reports_and_clears():
    kq.kq_device_errors()
    kq.kq_diag_wait_timeout(2_000_000)             # about a millisecond
    torch.cuda.synchronize()
    assert kq.kq_device_errors() == [0, 0, 0, 0, 1, 0]
    assert kq.kq_device_errors() == [0, 0, 0, 0, 0, 0]
    # the context stays usable
    x = torch.ones(4, 4096, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(4, 4096, dtype=torch.float32, device="cuda")
    kq.kq_rht(x, 0, None, out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
