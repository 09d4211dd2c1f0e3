"""The benchmark's multi-rank host logic on CPU: two gloo ranks (the N > 1
path of bench.py without a GPU).  Each rank draws its own batch, the step
time is the maximum over ranks, and the whole-job GB/s counts every rank's
bytes."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from hadamard_rotated_activation_b200 import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.WORKLOADS["c1"].with_tokens(4)
        inp = wl.make_inputs(w, seed=bench.rank_seed(w, rank))
        first = torch.tensor(inp.values[0, :8], dtype=torch.float64)
        rows = [torch.zeros_like(first) for _ in range(world)]
        dist.all_gather(rows, first)
        ms = 1.0 + 2.0 * rank                      # rank r "took" 1 + 2r ms
        got = bench.max_over_ranks(torch, dist, ms, torch.device("cpu"))
        out[rank] = (got, [r.numpy().tolist() for r in rows])
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_own_batches():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        assert res[r][0] == 3.0                     # the slowest rank's time, everywhere
    rows = res[0][1]
    assert rows == res[1][1]
    assert not np.allclose(rows[0], rows[1])       # the ranks' batches differ


def test_whole_job_rate_and_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_gbs(1e9, 4, 1000.0) == pytest.approx(4.0)
    assert bench.max_over_ranks(torch, None, 2.5, None) == 2.5
