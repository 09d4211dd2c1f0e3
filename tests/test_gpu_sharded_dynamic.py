"""GPU: the dynamic NVFP4 phases (KQ_DYN_STATS / KQ_DYN_EXACT / KQ_DYN_QUANT)
on row shards of one tensor, with the all-reduce(max) between the phases
done on the host (the shards run one after the other on one GPU; no kernel
waits for another), give bit for bit the codes, block scales and tensor
scale of the single dynamic call on the whole tensor, on every NVFP4 kernel
family and with an empty shard."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from hadamard_rotated_activation_b200 import workloads as wl
import hadamard_rotated_activation_b200 as kq
import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


@pytest.mark.parametrize("dim,block,splits", [
    (4096, 0, (300, 437)),        # 4096-wide tensor-core kernels
    (4096, 128, (500, 0, 200)),   # block-128 kernel, an empty shard
    (2048, 0, (100, 150)),        # warp per row
    (12288, 0, (7, 6)),           # row per CTA
])
def test_sharded_phases_equal_the_single_call(dim, block, splits):
    T = sum(splits)
    w = wl.Workload("c4", T, dim, wl.BF16, block, True, wl.NVFP4, 21)
    inp = wl.make_inputs(w)
    x, s = P.to_device(inp)
    c0, b0, t0, ws0 = kq.empty_nvfp4(T, dim, block)
    kq.kq_rht_quant_nvfp4(x, block, s, c0, b0, t0, ws0, dynamic=True)
    shards, r0 = [], 0
    for n in splits:
        shards.append((x[r0:r0 + n],) + kq.empty_nvfp4(n, dim, block))
        r0 += n

    def phase(flag):
        for xs, c, b, t, ws in shards:
            if xs.shape[0] > 0:
                kq.kq_rht_quant_nvfp4(xs, block, s, c, b, t, ws, dynamic=True, phases=flag)

    def all_reduce(lo, hi, dt):
        words = [ws.view(-1)[lo:hi].view(dt) for _, _, _, _, ws in shards]
        m = torch.stack(words).max(dim=0).values
        for wd in words:
            wd.copy_(m)

    for xs, c, b, t, ws in shards:
        if xs.shape[0] == 0:
            ws.view(-1)[0:16].zero_()
    phase(kq.KQ_DYN_STATS)
    all_reduce(0, 4, torch.int32)
    phase(kq.KQ_DYN_EXACT)
    all_reduce(8, 16, torch.int64)
    phase(kq.KQ_DYN_QUANT)
    torch.cuda.synchronize()
    nonempty = [sh for sh in shards if sh[0].shape[0] > 0]
    assert torch.equal(torch.cat([sh[1] for sh in nonempty]), c0)
    assert torch.equal(torch.cat([sh[2] for sh in nonempty]), b0)
    for sh in nonempty:
        assert sh[3].view(torch.int32).item() == t0.view(torch.int32).item()


def test_phase_flags_need_dynamic_mode():
    x = torch.zeros((4, 4096), dtype=torch.bfloat16, device="cuda")
    c, b, t, ws = kq.empty_nvfp4(4, 4096, 0)
    with pytest.raises(kq.KQError):
        kq.kq_rht_quant_nvfp4(x, 0, None, c, b, t, None, dynamic=False,
                              phases=kq.KQ_DYN_STATS)
