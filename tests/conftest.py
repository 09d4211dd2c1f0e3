import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")


def read_golden(name):
    """Non-comment, non-empty lines of a golden fixture, split on whitespace."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def golden():
    return read_golden


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Per-comparison parity counts of the GPU tests: rows and codes compared,
    scale mismatches (must be 0), code differences inside the 1e-5 boundary
    window (allowed, reported) and outside it (must be 0).  Also written as
    JSON to the file named by KQ_PARITY_REPORT, when set."""
    mod = sys.modules.get("parity")
    report = getattr(mod, "REPORT", None)
    if not report:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity counts (GPU vs oracle)")
    tr.write_line(f"{'comparison':34s} {'rows':>7s} {'codes':>11s} {'scales':>9s} "
                  f"{'scale!=':>7s} {'near':>5s} {'bad':>4s}")
    for name in sorted(report):
        c = report[name]
        tr.write_line(f"{name:34s} {c.rows:7d} {c.codes:11d} {c.scales:9d} "
                      f"{c.scale_mismatch:7d} {c.near:5d} {c.bad:4d}")
    path = os.environ.get("KQ_PARITY_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump({k: v.as_dict() for k, v in sorted(report.items())}, f, indent=1)
