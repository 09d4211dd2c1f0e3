"""bench.py reports an ncu DRAM-traffic figure only while the kernel's sources
are the ones it was captured on: the stored digest must equal the digest of
the kernel file and the shared headers, else the figure is withheld (None)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _tree(tmp_path):
    csrc = tmp_path / "hadamard_rotated_activation_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// kernel v1\n")
    (csrc / "h.cuh").write_text("// header v1\n")
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_follows_the_source_digest(tmp_path, monkeypatch):
    import bench
    csrc = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    entry = {"kernel": "k", "sources": ["k.cu", "h.cuh"], "dram_bytes_per_launch": 123456,
             "source_digest": bench.source_digest(["k.cu", "h.cuh"])}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"w": entry}))
    assert bench.ncu_traffic("w") == 123456.0
    assert bench.ncu_traffic("missing") is None
    (csrc / "h.cuh").write_text("// header v2\n")        # a shared header changed
    assert bench.ncu_traffic("w") is None
    (csrc / "h.cuh").write_text("// header v1\n")
    assert bench.ncu_traffic("w") == 123456.0
    (csrc / "k.cu").write_text("// kernel v2\n")         # the kernel changed
    assert bench.ncu_traffic("w") is None


def test_digest_depends_on_names_order_and_contents(tmp_path, monkeypatch):
    import bench
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d = bench.source_digest(["k.cu", "h.cuh"])
    assert len(d) == 16 and d == bench.source_digest(["k.cu", "h.cuh"])
    assert d != bench.source_digest(["h.cuh", "k.cu"])
    assert d != bench.source_digest(["k.cu"])


def test_committed_entries_name_existing_sources():
    import bench
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for key, e in d.items():
        assert e["dram_bytes_per_launch"] > 0, key
        for name in e["sources"]:
            assert os.path.exists(os.path.join(ROOT, "hadamard_rotated_activation_b200", "csrc",
                                               name)), (key, name)
        assert set(bench.KERNEL_HEADERS) <= set(e["sources"]), key


def test_dynamic_nvfp4_launch_counts():
    """The per-workload launch counts follow the library's dispatch: bf16
    block-128 rows up to 8192 run the dynamic scale in two kernels (the exact
    maximum inside the quantisation pass), other shapes in three."""
    import bench
    from hadamard_rotated_activation_b200 import workloads as wl
    counts = {}
    for key in ("c2", "c4"):
        w = wl.WORKLOADS[key]
        counts[key] = bench.make_step(None, None, w, None, None, None, "dynamic")[2]
    assert counts == {"c2": 2, "c4": 3}
    big = wl.WORKLOADS["c2"].with_tokens(8193)
    assert bench.make_step(None, None, big, None, None, None, "dynamic")[2] == 3
    assert bench.make_step(None, None, wl.WORKLOADS["c2"], None, None, None, "static")[2] == 1
