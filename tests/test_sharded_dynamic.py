"""The sharded dynamic NVFP4 protocol on CPU ranks (gloo): rows split over
two or three ranks, one of them possibly empty; each rank runs the protocol
of the library's Python binding (phase 1, all-reduce(max) of the lower
bound, phase 2, all-reduce(max) of the exact maximum, phase 3), with the
three phases emulated by the oracle on the rank's rows.  Every rank must end
with the tensor scale of the whole tensor: the oracle's single-tensor
result.  (QuaRot reviews, final comments: RHT per batch of data is data
parallelism; the tensor scale is a property of the whole tensor.)"""
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


def _emulated_phases(rows, signs, block, lower, gmax, state, rel_err=2.0 ** -20):
    """run_phase for one rank: the oracle's exact row maxima with an error
    bound of rel_err of each (a stand-in for the kernels' fp32 bound)."""
    import oracle
    from hadamard_rotated_activation_b200 import KQ_DYN_STATS, KQ_DYN_EXACT, KQ_DYN_QUANT

    def run(flag):
        if flag == KQ_DYN_STATS:
            s = np.abs(oracle.rht_unnormalized(rows, signs, block)).max(axis=1)
            state["rowmax"] = s
            state["E"] = s * rel_err
            low = np.float32(np.max(s - state["E"]))
            lower.copy_(torch.tensor([np.array([low]).view(np.int32)[0]], dtype=torch.int32))
        elif flag == KQ_DYN_EXACT:
            L = np.array([int(lower.item())], dtype=np.int32).view(np.float32)[0]
            cand = state["rowmax"] + state["E"] >= np.float64(L)
            state["candidates"] = int(cand.sum())
            g = float(state["rowmax"][cand].max()) if cand.any() else 0.0
            gmax.copy_(torch.tensor([np.array([g]).view(np.int64)[0]], dtype=torch.int64))
        elif flag == KQ_DYN_QUANT:
            g = np.array([int(gmax.item())], dtype=np.int64).view(np.float64)[0]
            n = rows.shape[1] if block == 0 else block
            state["t"] = np.float32(g / np.sqrt(np.float64(n)) / 2688.0)
    return run


def _rank_main(rank, world, port, splits, out):
    sys.path.insert(0, ROOT)
    from hadamard_rotated_activation_b200 import sharded_dynamic_protocol
    from hadamard_rotated_activation_b200 import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = wl.make_inputs(wl.WORKLOADS["c4"].with_tokens(sum(splits)), seed=5)
        r0 = sum(splits[:rank])
        rows = inp.values[r0:r0 + splits[rank]]
        lower = torch.zeros(1, dtype=torch.int32)
        gmax = torch.zeros(1, dtype=torch.int64)
        state = {}
        run = _emulated_phases(rows, inp.signs, 0, lower, gmax, state)
        sharded_dynamic_protocol(run, lower, gmax,
                                 lambda t: dist.all_reduce(t, op=dist.ReduceOp.MAX),
                                 rows.shape[0] == 0)
        out[rank] = (float(state.get("t", np.nan)), state.get("candidates", 0),
                     splits[rank])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("splits", [(7, 9), (16, 0), (5, 6, 4)])
def test_every_rank_gets_the_whole_tensor_scale(splits):
    import oracle
    from hadamard_rotated_activation_b200 import workloads as wl
    world = len(splits)
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), splits, out), nprocs=world, join=True)
    inp = wl.make_inputs(wl.WORKLOADS["c4"].with_tokens(sum(splits)), seed=5)
    t_ref = oracle.nvfp4_tensor_scale(oracle.rht(inp.values, inp.signs, 0))
    for r in range(world):
        t, cand, nrows = out[r]
        if nrows == 0:
            continue                                   # an empty rank quantizes nothing
        assert np.float32(t) == t_ref, (r, t, t_ref)
    # the global maximum row is a candidate on exactly the rank that holds it
    assert sum(out[r][1] for r in range(world)) >= 1
