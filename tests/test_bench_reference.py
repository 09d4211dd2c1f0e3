"""bench.py --impl reference on CPU: the oracle arm prints one JSON line with
the keys the benchmark contract asks for, and only rank 0 prints.  The row
sample is cut to two rows so that the test takes about a second."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

KEYS = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e")


@pytest.mark.parametrize("workload", ["c1", "c4"])
def test_reference_arm_json_line(workload, monkeypatch, capsys):
    import bench
    monkeypatch.setattr(bench, "cpu_sample_rows", lambda *a, **k: 2)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", workload,
                                      "--steps", "1", "--warmup", "1"])
    args = bench.parse_args()
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in KEYS:
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith(workload)
    assert line["config"]["sample_rows"] == 2


def test_reference_arm_other_ranks_print_nothing(monkeypatch, capsys):
    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1",
                                      "--warmup", "1"])
    bench.run_reference(bench.parse_args(), 1, 2)
    assert capsys.readouterr().out == ""


def test_sample_parity_counts_on_cpu():
    """The parity counts the CPU-baseline leg attaches to the bench line: the
    oracle's own outputs give zero mismatches; a flipped scale is counted."""
    import numpy as np
    import bench
    import oracle
    from hadamard_rotated_activation_b200 import workloads as wl

    samples = {}
    for key in ("c1", "c5", "c4"):
        w = wl.WORKLOADS[key].with_tokens(3)
        inp = wl.make_inputs(w)
        y = oracle.rht(inp.values, inp.signs, w.block)
        t = None
        if w.fmt == wl.INT4_SYM:
            q, s = oracle.int4_sym_per_token(y)
            got = (oracle.pack_nibbles(q), s)
        elif w.fmt == wl.INT4_ASYM:
            u, s, z = oracle.int4_asym_group(y, w.group)
            got = (oracle.pack_nibbles(u), s, z)
        else:
            c, b, t = oracle.nvfp4(y)
            got = (oracle.pack_nibbles(c), b)
        samples[key] = {"workload": w, "values": inp.values, "signs": inp.signs, "got": got,
                        "tensor_scale": t}
    out = bench.sample_parity(oracle, wl, samples)
    for key, c in out.items():
        assert c["rows"] == 3 and c["scale_mismatch"] == 0 and c["bad"] == 0, (key, c)
    b = samples["c4"]["got"][1].copy()
    b[0, 0] ^= 1
    samples["c4"]["got"] = (samples["c4"]["got"][0], b)
    assert bench.sample_parity(oracle, wl, {"c4": samples["c4"]})["c4"]["scale_mismatch"] >= 1
