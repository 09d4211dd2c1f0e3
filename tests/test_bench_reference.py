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
