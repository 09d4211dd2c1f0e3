#!/usr/bin/env python
"""Benchmark: rotated + quantized GB/s and tokens/s on B200, fraction of HBM peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c4]
                    [--impl kq|reference] [--no-extras] [--roundtrip-only]

A step is one pass of the hot path over one batch of the workload: load +
sign, Hadamard butterflies, normalisation folded into the scales, extrema,
exact scales, 4-bit rounding, nibble packing and stores.  The default
workload is the 16384 x 4096 bf16 batch with a full-row Hadamard and NVFP4
output (static fp32 tensor scale, computed once by the dynamic path during
warm-up; the dynamic two-pass time is reported alongside).

Inputs are resident in HBM before the timed region; consecutive steps cycle
through enough independent buffer sets that every step reads its input from
DRAM (the sets together exceed three times the 126 MB L2), so no L2 flush is
needed between steps.  Times come from CUDA events on the launching stream;
for N > 1 every rank times its own batch (weak scaling, no data-path
collective) and the maximum over ranks is reported.

`--impl reference` times the CPU oracle (fp64 dense D.H product + scalar
quantizer) on the host cores over a bounded sample of rows per step.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
# The headline metric: GB/s of algorithmic bytes (input read + codes and scales
# written), with tokens/s and the fraction of the measured HBM peak alongside.
METRIC = "rotated+quantized GB/s and tokens/s at 1 B200; fraction of HBM peak"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="c4")
    p.add_argument("--tokens", type=int, default=0,
                   help="override the workload's row count (small cases for profiling)")
    p.add_argument("--impl", default="kq", choices=["kq", "reference"])
    p.add_argument("--no-extras", action="store_true",
                   help="skip the per-workload table, dynamic and round-trip timings")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--roundtrip-only", action="store_true",
                   help="time only the c4 dequant + inverse round trip (one JSON line)")
    p.add_argument("--gemm-only", action="store_true",
                   help="time only the NVFP4 GEMM consumer of the c4 batch (one JSON line; "
                        "--tokens sets M)")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle baseline sample")
    return p.parse_args()


# ------------------------------------------------------------------ peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_HEADERS = ("kq_sm100.cuh", "kq_device.cuh", "kq_internal.h")
# B200 HBM3e datasheet bandwidth (DGX figure), a second denominator beside the
# measured copy peak
DATASHEET_HBM_GBS = 8000.0


def source_digest(files):
    """Digest of the named csrc files (name and contents), in order."""
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "hadamard_rotated_activation_b200", "csrc", name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel's current sources (its .cu file and the shared headers); else
    None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel_key]
        if e.get("source_digest") != source_digest(e["sources"]):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, torch_device):
        self.ok = False
        self.samples = []
        self.busy = []          # samples taken while the GPU reported activity
        self.reasons = 0
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            h = None
            try:
                import torch
                props = torch.cuda.get_device_properties(torch_device)
                bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id,
                                            props.pci_device_id)
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def sample(self):
        if not self.ok:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
            self.samples.append(mhz)
            if util > 0:
                self.busy.append(mhz)
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def start(self, period_s=0.02):
        """Samples every period_s on a thread until stop()."""
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                self.sample()
                self._stop.wait(period_s)
        self._thr = threading.Thread(target=run, daemon=True)
        self._thr.start()
        return self

    def stop(self):
        if getattr(self, "_thr", None) is not None:
            self._stop.set()
            self._thr.join()
            self._thr = None

    def summary(self):
        names = [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1]
        load = self.busy if self.busy else self.samples
        return {
            "sm_mhz": statistics.median(load) if load else None,
            "sm_max_mhz": self.max_mhz,
            "reasons": names,
            "samples": len(self.samples),
            "samples_under_load": len(self.busy),
            "source": "nvml, sampled every 20 ms from the first warm-up step to the end "
                      "of the per-workload table",
        }


# ------------------------------------------------------------- workloads
def make_step(torch, kq, w, dev_inputs, signs, tensor_scale=None, mode="static"):
    """Returns (make_set, step(set), kernel launches per step)."""
    from hadamard_rotated_activation_b200 import workloads as wl
    t, n, b = w.tokens, w.dim, w.block

    if w.fmt == "nvfp4":
        def make_set(x):
            c, bs, ts, ws = kq.empty_nvfp4(t, n, b)
            if tensor_scale is not None:
                ts.fill_(float(tensor_scale))
            return (x, c, bs, ts, ws)

        if mode == "static":
            def step(s):
                kq.kq_rht_quant_nvfp4(s[0], b, signs, s[1], s[2], s[3], None, dynamic=False)
            launches = 1
        else:
            def step(s):
                kq.kq_rht_quant_nvfp4(s[0], b, signs, s[1], s[2], s[3], s[4], dynamic=True)
            # statistics, exact maximum, quantization; bf16 block-128 rows up
            # to 8192 run the last two in one launch (the workspace clear is a
            # memset, not a kernel)
            launches = 2 if (b == 128 and w.dtype == wl.BF16 and t <= 8192) else 3
    elif w.fmt == "int4_sym":
        def make_set(x):
            return (x,) + kq.empty_int4_sym(t, n)

        def step(s):
            kq.kq_rht_quant_int4(s[0], b, signs, 0, False, s[1], s[2])
        launches = 1
    else:
        def make_set(x):
            return (x,) + kq.empty_int4_asym(t, n, w.group)

        def step(s):
            kq.kq_rht_quant_int4(s[0], b, signs, w.group, True, s[1], s[2], s[3])
        launches = 1
    return make_set, step, launches


def device_input(torch, inp, wl, dev):
    import numpy as np
    if inp.workload.dtype == wl.BF16:
        return torch.from_numpy(inp.stored.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(inp.stored).to(dev)


def n_sets(bytes_per_set):
    return max(2, -(-3 * L2_BYTES // max(bytes_per_set, 1)))


def time_steps(torch, step, sets, k, warmup, sampler=None, stream=None):
    for i in range(warmup):
        step(sets[i % len(sets)])
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(k):
        step(sets[i % len(sets)])
    end.record(stream)
    if sampler is not None:
        while not end.query():
            sampler.sample()
            time.sleep(0.0002)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


# -------------------------------------------------------------- CPU oracle
def oracle_step(oracle_mod, wl, inp_rows, w):
    y = oracle_mod.rht(inp_rows.values, inp_rows.signs, w.block)
    if w.fmt == wl.NVFP4:
        oracle_mod.nvfp4(y)
    elif w.fmt == wl.INT4_SYM:
        oracle_mod.int4_sym_per_token(y)
    else:
        oracle_mod.int4_asym_group(y, w.group)


def cpu_sample_rows(oracle_mod, wl, w, seconds):
    """Rows of the workload the oracle handles in about `seconds`."""
    probe = wl.make_inputs(w, tokens=4)
    oracle_step(oracle_mod, wl, probe, w)          # builds and caches H
    t0 = time.perf_counter()
    oracle_step(oracle_mod, wl, probe, w)
    per_row = max((time.perf_counter() - t0) / 4, 1e-6)
    return int(max(4, min(w.tokens, seconds / per_row)))


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def sample_outputs(w, inp, out_set, tscale, rows=256):
    """The first `rows` rows of a timed step's inputs and outputs, on the host,
    for the parity counts of the CPU-baseline leg."""
    import numpy as np
    r = min(rows, w.tokens)
    return {"workload": w.with_tokens(r), "values": inp.values[:r], "signs": inp.signs,
            "got": tuple(t[:r].cpu().numpy() for t in out_set[1:]
                         if hasattr(t, "dim") and t.dim() >= 1 and t.shape[0] == w.tokens),
            "tensor_scale": None if tscale is None else np.float32(tscale)}


def sample_parity(oracle_mod, wl, samples):
    """Counts of the sampled rows against the oracle: rows, codes, scales,
    scale mismatches (must be 0), code differences within the 1e-5 boundary
    window (reported) and outside it (must be 0).  NVFP4 is checked under the
    timed call's own tensor scale."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity as P
    out = {}
    for name, smp in samples.items():
        w = smp["workload"]
        y = oracle_mod.rht(smp["values"], smp["signs"], w.block)
        g = smp["got"]
        if w.fmt == wl.NVFP4:
            t = smp["tensor_scale"]
            c = P.check_nvfp4(g[0], g[1], t, y, tensor_scale=t, strict=False, name=False)
        elif w.fmt == wl.INT4_SYM:
            c = P.check_int4_sym(g[0], g[1], y, strict=False, name=False)
        else:
            c = P.check_int4_asym(g[0], g[1], g[2], y, w.group, strict=False, name=False)
        out[name] = c.as_dict()
    return out


def run_cpu_baseline(w, seconds, samples=None):
    """The oracle timed on the host cores over a bounded sample of rows, and
    (when `samples` holds GPU outputs) the parity counts of those outputs."""
    import oracle as oracle_mod
    from hadamard_rotated_activation_b200 import workloads as wl
    rows = cpu_sample_rows(oracle_mod, wl, w, seconds)
    inp = wl.make_inputs(w, tokens=rows)
    t0 = time.perf_counter()
    oracle_step(oracle_mod, wl, inp, w)
    dt = time.perf_counter() - t0
    wb = w.with_tokens(rows)
    base = {
        "value": round(wb.algorithmic_bytes() / dt / 1e9, 6),
        "unit": "GB/s",
        "tokens_per_s": round(rows / dt, 3),
        "cores": cpu_threads(),
        "kind": "oracle",
        "sample": f"{rows} of {w.tokens} rows of workload {w.key} "
                  f"(fp64 dense D.H + scalar quantizer), {dt:.2f} s wall",
    }
    par = None
    if samples:
        par = {"rows_per_workload": "the first 256 rows of each timed call's output",
               "counts": sample_parity(oracle_mod, wl, samples)}
    return base, par


# ------------------------------------------------------------ multi-rank
def rank_seed(w, rank):
    """Seed of rank `rank`'s batch: every rank draws its own (weak scaling)."""
    return w.seed + 1000 * rank


def max_over_ranks(torch, dist, value, device):
    """The maximum of a per-rank float over all ranks (the job's time is the
    slowest rank's); `value` itself without a process group."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank, world, ms_per_step):
    """GB/s of the whole job: every rank moves bytes_per_rank per step, and
    the step lasts ms_per_step (the slowest rank's)."""
    return bytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle, timed on the host cores."""
    if rank != 0:
        return
    import oracle as oracle_mod
    from hadamard_rotated_activation_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_tokens(args.tokens)
    per_step_s = max(2.0, min(20.0, 150.0 / max(args.steps + args.warmup, 1)))
    rows = cpu_sample_rows(oracle_mod, wl, w, per_step_s)
    inp = wl.make_inputs(w, tokens=rows)
    for _ in range(args.warmup):
        oracle_step(oracle_mod, wl, inp, w)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(oracle_mod, wl, inp, w)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    wb = w.with_tokens(rows)
    gbs = wb.algorithmic_bytes() / dt / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(gbs, 6), "unit": "GB/s", "n_gpus": 0, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, forward_only=True, sample_rows=rows),
        "tokens_per_s": round(rows / dt, 3),
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": cpu_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {w.tokens} rows per step"},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, forward_only=False, **extra):
    desc = w.description
    if forward_only and "; dequant + inverse round trip" in desc:
        desc = desc.replace("; dequant + inverse round trip", "") + \
            " (timed step: the forward rotation + quantization; the dequant + inverse " \
            "round trip is timed separately, per_workload.c4_roundtrip)"
    d = {
        "workload": f"{w.key}: {desc}",
        "tokens": w.tokens, "dim": w.dim, "block": w.block,
        "input_dtype": w.dtype, "format": w.fmt, "seed": w.seed,
        "global_batch": w.tokens, "seq_len": None, "parallelism": "dp (independent batches)",
    }
    d.update(extra)
    return d


# ------------------------------------------------------------------ main
def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import numpy as np
    import torch
    import hadamard_rotated_activation_b200 as kq
    from hadamard_rotated_activation_b200 import workloads as wl

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    kq.lib()

    w = wl.WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_tokens(args.tokens)
    peak, peak_kind = measured_peaks()
    if args.roundtrip_only:
        if rank == 0:
            print(json.dumps(roundtrip(torch, kq, wl, dev, peak, args.steps, args.warmup,
                                       args.tokens)), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return
    if args.gemm_only:
        if rank == 0:
            inp = wl.make_inputs(w)
            x0 = device_input(torch, inp, wl, dev)
            sg = torch.from_numpy(inp.signs).to(dev)
            print(json.dumps({"c4_gemm_consumer": gemm_consumer(torch, kq, wl, dev, x0, sg,
                                                                 args.steps)}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return
    # every rank draws its own batch (weak scaling)
    inp = wl.make_inputs(w, seed=rank_seed(w, rank))
    x0 = device_input(torch, inp, wl, dev)
    signs = None if inp.signs is None else torch.from_numpy(inp.signs).to(dev)

    # tensor scale for the static NVFP4 step: the dynamic path's own result
    tscale = None
    if w.fmt == wl.NVFP4:
        c, bs, ts, ws = kq.empty_nvfp4(w.tokens, w.dim, w.block)
        kq.kq_rht_quant_nvfp4(x0, w.block, signs, c, bs, ts, ws, dynamic=True)
        torch.cuda.synchronize()
        tscale = float(ts.item())
        del c, bs, ts, ws

    make_set, step, launches = make_step(torch, kq, w, None, signs, tscale, "static")
    set_bytes = w.algorithmic_bytes()
    sets = [make_set(x0 if i == 0 else x0.clone()) for i in range(n_sets(set_bytes))]

    sampler = ClockSampler(dev).start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ms = time_steps(torch, step, sets, args.steps, args.warmup, None, stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = max_over_ranks(torch, dist, ms, dev)
    ms_step = ms / max(args.steps, 1)
    alg = w.algorithmic_bytes()
    gbs_rank = alg / (ms_step * 1e-3) / 1e9
    value = whole_job_gbs(alg, world, ms_step)
    tokens_s = w.tokens * world / (ms_step * 1e-3)

    # ---- end to end through the public API: pinned host in, host out.  Rows
    # are independent (static tensor scale), so the batch goes through in
    # chunks on three streams: the copy in of chunk i + 1 and the copy out of
    # chunk i - 1 overlap the call on chunk i (both link directions at once).
    x_host = torch.from_numpy(inp.stored.view(np.int16) if w.dtype == wl.BF16
                              else inp.stored).pin_memory()
    e2e_set = make_set(torch.empty_like(x0))
    out_idx = (1, 2, 3) if w.fmt == wl.INT4_ASYM else (1, 2)
    outs_host = [torch.empty(e2e_set[i].shape, dtype=e2e_set[i].dtype).pin_memory()
                 for i in out_idx]
    in_bytes = x_host.numel() * x_host.element_size()
    out_bytes = sum(o.numel() * o.element_size() for o in outs_host)
    n_chunks = 8 if w.tokens >= 8 * 256 else 1
    bounds = [(w.tokens * i // n_chunks, w.tokens * (i + 1) // n_chunks)
              for i in range(n_chunks)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))

    def rows(tensor, r0, r1):
        if torch.is_tensor(tensor) and tensor.dim() >= 1 and tensor.shape[0] == w.tokens:
            return tensor[r0:r1]
        return tensor

    def e2e_step(_s):
        main = torch.cuda.current_stream()
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(main)
        dst = e2e_set[0].view(torch.int16) if w.dtype == wl.BF16 else e2e_set[0]
        for r0, r1 in bounds:
            with torch.cuda.stream(s_in):
                dst[r0:r1].copy_(x_host[r0:r1], non_blocking=True)
            s_cmp.wait_stream(s_in)
            with torch.cuda.stream(s_cmp):
                step(tuple(rows(t, r0, r1) for t in e2e_set))
            s_out.wait_stream(s_cmp)
            with torch.cuda.stream(s_out):
                for h, i in zip(outs_host, out_idx):
                    h[r0:r1].copy_(e2e_set[i][r0:r1], non_blocking=True)
        main.wait_stream(s_out)

    k_e2e = max(3, min(args.steps, 50))
    ms_e2e = time_steps(torch, e2e_step, [None], k_e2e, max(3, min(args.warmup, 5)))
    # the chunked path must give the device-resident path's result, every
    # output (codes, scales and, for asymmetric INT4, zero points)
    for h, i in zip(outs_host, out_idx):
        if not torch.equal(h, sets[0][i].cpu()):
            raise SystemExit(f"end-to-end output {i} differs from the device-resident step")
    ms_e2e = max_over_ranks(torch, dist, ms_e2e, dev)
    e2e_gbs = whole_job_gbs(alg, world, ms_e2e / k_e2e)

    kernel_key = f"{w.key}_{w.fmt}_static" if w.fmt == wl.NVFP4 else f"{w.key}_{w.fmt}"
    traffic = ncu_traffic(kernel_key)
    line = {
        "metric": METRIC,
        "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, forward_only=True,
                                  l2="inputs larger than L2: %d rotating buffer sets"
                                  % len(sets),
                                  tensor_scale="static: an input of the timed call, computed "
                                  "once beforehand by the dynamic path (the dynamic two-pass "
                                  "call is timed as dynamic_tensor_scale)"
                                  if w.fmt == wl.NVFP4 else None),
        "tokens_per_s": round(tokens_s, 1),
        "frac_of_hbm_peak": round(gbs_rank / peak, 4),
        "frac_of_datasheet_hbm": round(gbs_rank / DATASHEET_HBM_GBS, 4),
        "gpu_launches": launches * args.steps,
        "roofline": {
            "bound": "hbm", "achieved": round(gbs_rank, 3), "peak": peak, "unit": "GB/s",
            "frac": round(gbs_rank / peak, 4), "peak_kind": peak_kind,
            "traffic": None if traffic is None else round(traffic),
            "kernel": kernel_key,
            "bytes_per_launch": alg,
        },
        "e2e": {"value": round(e2e_gbs, 3), "unit": "GB/s",
                "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
                "ms_per_step": round(ms_e2e / k_e2e, 4), "chunks": n_chunks,
                "streams": "copy in / call / copy out"},
    }

    samples = {"headline": sample_outputs(w, inp, sets[0], tscale)}
    if not args.no_extras and rank == 0:
        line["per_workload"], more = extras(torch, kq, wl, dev, peak, args)
        samples.update(more)
        dyn = line["per_workload"].get(f"{w.key}_dynamic")
        if dyn is not None:
            line["dynamic_tensor_scale"] = {k: dyn[k] for k in ("ms", "GB/s", "frac",
                                                                 "launches_per_step")}
    sampler.stop()
    line["clocks"] = sampler.summary()
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        line["cpu_baseline"], line["parity"] = run_cpu_baseline(w, args.cpu_seconds, samples)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def extras(torch, kq, wl, dev, peak, args):
    """Per-workload forward timings (all five), NVFP4 dynamic, and the c4
    dequant + inverse round trip.  Not part of the headline value."""
    import numpy as np
    out, samples = {}, {}
    k = max(20, min(args.steps, 200))
    for key, w in wl.WORKLOADS.items():
        inp = wl.make_inputs(w)
        x0 = device_input(torch, inp, wl, dev)
        signs = None if inp.signs is None else torch.from_numpy(inp.signs).to(dev)
        modes = ["static", "dynamic"] if w.fmt == wl.NVFP4 else ["-"]
        tscale = None
        if w.fmt == wl.NVFP4:
            c, bs, ts, ws = kq.empty_nvfp4(w.tokens, w.dim, w.block)
            kq.kq_rht_quant_nvfp4(x0, w.block, signs, c, bs, ts, ws, dynamic=True)
            torch.cuda.synchronize()
            tscale = float(ts.item())
        for mode in modes:
            make_set, step, launches = make_step(torch, kq, w, None, signs, tscale,
                                                 mode if mode != "-" else "static")
            nset = n_sets(w.algorithmic_bytes())
            sets = [make_set(x0 if i == 0 else x0.clone()) for i in range(nset)]
            ms = time_steps(torch, step, sets, k, 5) / k
            alg = w.algorithmic_bytes()
            gbs = alg / (ms * 1e-3) / 1e9
            name = key if mode == "-" else f"{key}_{mode}"
            out[name] = {"ms": round(ms, 5), "GB/s": round(gbs, 2),
                         "frac": round(gbs / peak, 4),
                         "tokens_per_s": round(w.tokens / (ms * 1e-3), 1),
                         "launches_per_step": launches,
                         "bytes": alg}
            tkey = f"{key}_{w.fmt}" + ("_static" if mode == "static" else "")
            if mode != "dynamic" and ncu_traffic(tkey) is not None:
                out[name]["traffic"] = round(ncu_traffic(tkey))
            t_used = None
            if w.fmt == wl.NVFP4:
                t_used = float(sets[0][3].item())
            samples[name] = sample_outputs(w, inp, sets[0], t_used)
            del sets
        if key == "c4":
            out.update(roundtrip(torch, kq, wl, dev, peak, k, 5, 0, x0, signs))
            out["c4_gemm_consumer"] = gemm_consumer(torch, kq, wl, dev, x0, signs, k)
            # the same batch as MXFP4 (E8M0 scale per 32 elements)
            mx_sets = [(x0 if i == 0 else x0.clone(),) + kq.empty_mxfp4(w.tokens, w.dim)
                       for i in range(n_sets(w.tokens * w.dim * 2))]

            def mx_step(st):
                kq.kq_rht_quant_mxfp4(st[0], w.block, signs, st[1], st[2])
            ms = time_steps(torch, mx_step, mx_sets, k, 5) / k
            mb = w.tokens * (w.dim * 2 + w.dim // 2 + w.dim // 32)
            out["c4_mxfp4"] = {"ms": round(ms, 5), "GB/s": round(mb / (ms * 1e-3) / 1e9, 2),
                               "frac": round(mb / (ms * 1e-3) / 1e9 / peak, 4), "bytes": mb,
                               "tokens_per_s": round(w.tokens / (ms * 1e-3), 1),
                               "launches_per_step": 1}
            del mx_sets
        del x0
        torch.cuda.empty_cache()
    return out, samples


def fp4_peak_tflops():
    """Dense FP4 tensor peak: the measured bf16 GEMM burst figure times the
    nominal FP4 / bf16 ratio (9 / 2.25 = 4), or the fallback bf16 figure x 4."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return 4.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 4"
    except Exception:
        return 4.0 * 1590.0, "fallback bf16 x 4"


def gemm_consumer(torch, kq, wl, dev, x0, signs, k):
    """The 4-bit GEMM that consumes the c4 batch: its rotated NVFP4 codes
    (static tensor scale, block scales in the tensor-core layout) times a
    4096 x 4096 weight rotated and quantized by the same call, fp32 out.  One
    launch per step; the 268 MB output exceeds the L2 on every step."""
    import numpy as np
    t, n = x0.shape
    rng = np.random.default_rng(44)
    wt = wl.round_to_bf16(rng.standard_normal((n, n)) / np.sqrt(n))
    wdev = torch.from_numpy(wl.bf16_bits(wt).view(np.int16)).to(dev).view(torch.bfloat16)
    ops = []
    for src, rows in ((x0, t), (wdev, n)):
        c0, b0, t0, ws = kq.empty_nvfp4(rows, n, 0)
        kq.kq_rht_quant_nvfp4(src, 0, signs, c0, b0, t0, ws, dynamic=True)
        cm, bm, tm, _ = kq.empty_nvfp4(rows, n, 0, mma_layout=True)
        tm.copy_(t0)
        kq.kq_rht_quant_nvfp4(src, 0, signs, cm, bm, tm, None, dynamic=False, mma_layout=True)
        ops.append((cm, bm, tm))
    (ca, sa, ta), (cb, sb, tb) = ops
    outs = [torch.empty((t, n), dtype=torch.float32, device=dev) for _ in range(2)]

    def step(o):
        kq.kq_gemm_nvfp4(ca, sa, ta, cb, sb, tb, o)
    kk = max(5, min(k, 50))
    ms = time_steps(torch, step, outs, kk, 3) / kk
    flops = 2.0 * t * n * n
    tf = flops / (ms * 1e-3) / 1e12
    peak, kind = fp4_peak_tflops()
    return {"ms": round(ms, 5), "TFLOP/s": round(tf, 1), "frac": round(tf / peak, 4),
            "shape": f"M={t} N={n} K={n}", "flops": flops, "launches_per_step": 1,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(peak, 1),
                         "unit": "TFLOP/s", "frac": round(tf / peak, 4), "peak_kind": kind,
                         "traffic": None}}


def roundtrip(torch, kq, wl, dev, peak, k, warmup, tokens=0, x0=None, signs=None):
    """The c4 round trip: NVFP4 codes of the batch, dequantized and rotated back
    to fp32 by the fused call (one launch), and by the two calls (dequant, then
    inverse rotation) for comparison; code sets rotate over 3x the L2."""
    w = wl.WORKLOADS["c4"]
    if tokens:
        w = w.with_tokens(tokens)
    if x0 is None:
        inp = wl.make_inputs(w)
        x0 = device_input(torch, inp, wl, dev)
        signs = None if inp.signs is None else torch.from_numpy(inp.signs).to(dev)
    c, bs, ts, ws = kq.empty_nvfp4(w.tokens, w.dim, w.block)
    kq.kq_rht_quant_nvfp4(x0, w.block, signs, c, bs, ts, ws, dynamic=True)
    in_bytes = w.tokens * w.dim // 2 + w.tokens * w.dim // 16
    code_sets = [(c, bs)] + [(c.clone(), bs.clone()) for _ in range(n_sets(in_bytes) - 1)]
    back = torch.empty((w.tokens, w.dim), dtype=torch.float32, device=dev)

    def rt(cs):
        kq.kq_dequant_rht_inverse(kq.KQ_FMT_NVFP4, cs[0], cs[1], None, ts, w.tokens,
                                  w.dim, w.block, 0, signs, back)
    ms = time_steps(torch, rt, code_sets, k, warmup) / k
    rbytes = in_bytes + 4 * w.tokens * w.dim
    gbs = rbytes / (ms * 1e-3) / 1e9
    out = {"c4_roundtrip": {"ms": round(ms, 5), "GB/s": round(gbs, 2),
                            "frac": round(gbs / peak, 4), "bytes": rbytes,
                            "tokens_per_s": round(w.tokens / (ms * 1e-3), 1),
                            "launches_per_step": 1}}
    if ncu_traffic("c4_roundtrip") is not None and not tokens:
        out["c4_roundtrip"]["traffic"] = round(ncu_traffic("c4_roundtrip"))
    back16 = torch.empty((w.tokens, w.dim), dtype=torch.bfloat16, device=dev)

    def rt16(cs):
        kq.kq_dequant_rht_inverse(kq.KQ_FMT_NVFP4, cs[0], cs[1], None, ts, w.tokens,
                                  w.dim, w.block, 0, signs, back16)
    ms16 = time_steps(torch, rt16, code_sets, k, warmup) / k
    b16 = in_bytes + 2 * w.tokens * w.dim
    g16 = b16 / (ms16 * 1e-3) / 1e9
    out["c4_roundtrip_bf16"] = {"ms": round(ms16, 5), "GB/s": round(g16, 2),
                                "frac": round(g16 / peak, 4), "bytes": b16,
                                "tokens_per_s": round(w.tokens / (ms16 * 1e-3), 1),
                                "launches_per_step": 1}
    del back16
    deq = torch.empty_like(back)

    def rt2(cs):
        kq.kq_dequant(kq.KQ_FMT_NVFP4, cs[0], cs[1], None, ts, w.tokens, w.dim, 0, deq)
        kq.kq_rht(deq, w.block, signs, back, inverse=True)
    k2 = max(3, min(k, 20))
    ms2 = time_steps(torch, rt2, code_sets, k2, min(warmup, 3)) / k2
    out["c4_roundtrip_two_calls"] = {"ms": round(ms2, 5), "launches_per_step": 2}
    return out


if __name__ == "__main__":
    main()
