"""GPU parity: the CUDA path through the C ABI vs the CPU oracle.

Small cases span several CTAs and a ragged row count, plus degenerate rows
(zeros, a single spike, constant, alternating, tiny, huge).  Full-size cases
run each workload at its published size in the launch configuration the
benchmark times and compare every row (in row chunks on the CPU); the
counts of every comparison, near-boundary code differences included, are
printed at the end of the session.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from hadamard_rotated_activation_b200 import workloads as wl
import hadamard_rotated_activation_b200 as kq
import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


def small_inputs(key, tokens, with_edges=True):
    w = wl.WORKLOADS[key]
    inp = wl.make_inputs(w, tokens=tokens)
    if not with_edges:
        return inp
    edges = wl.edge_rows(w.dim, w.dtype)
    vals = np.concatenate([inp.values, edges])
    return P.inputs_from_values(w, vals, inp.signs)


# ------------------------------------------------------------- rotation
@pytest.mark.parametrize("key,tokens", [("c1", 37), ("c2", 37), ("c3", 13), ("c4", 37),
                                        ("c5", 37)])
def test_rotation_forward_and_inverse(key, tokens):
    inp = small_inputs(key, tokens)
    w = inp.workload
    y_ref = oracle.rht(inp.values, inp.signs, w.block)
    y = P.gpu_rht(inp)
    P.check_rotation(y, y_ref)
    # inverse of the oracle's rotated values (fed as fp32)
    y32 = y_ref.astype(np.float32)
    winv = wl.Workload(w.key, w.tokens, w.dim, wl.F32, w.block, w.use_signs, w.fmt, w.seed)
    inv_inp = wl.Inputs(winv, y32.astype(np.float64), y32, inp.signs)
    x_back = P.gpu_rht(inv_inp, inverse=True)
    P.check_rotation(x_back, oracle.rht_inverse(y32.astype(np.float64), inp.signs, w.block))


@pytest.mark.parametrize("dim,block,dtype", [
    (32, 16, wl.BF16), (256, 32, wl.F32), (256, 0, wl.BF16), (384, 0, wl.BF16),
    (768, 0, wl.F32), (1024, 64, wl.BF16), (16384, 0, wl.BF16), (8192, 256, wl.F32),
    (12288, 1024, wl.BF16),
])
def test_rotation_other_shapes(dim, block, dtype):
    rng = np.random.default_rng(dim + block)
    x = rng.standard_normal((9, dim)) * rng.lognormal(0, 1, dim)
    x = wl.round_to_bf16(x) if dtype == wl.BF16 else x.astype(np.float32).astype(np.float64)
    s = (1 - 2 * rng.integers(0, 2, dim)).astype(np.int8)
    w = wl.Workload("x", 9, dim, dtype, block, True, wl.INT4_SYM, 0)
    inp = P.inputs_from_values(w, x, s)
    P.check_rotation(P.gpu_rht(inp), oracle.rht(x, s, block))
    y = oracle.rht(x, s, block)
    q, sc = P.gpu_int4_sym(inp)
    P.check_int4_sym(q, sc, y)
    codes, bs, ts = P.gpu_nvfp4(inp)
    P.check_nvfp4(codes, bs, ts, y)
    mc, ms = P.gpu_mxfp4(inp)
    P.check_mxfp4(mc, ms, y)


# ---------------------------------------------------------------- INT4
@pytest.mark.parametrize("key,tokens", [("c1", 37), ("c3", 13)])
def test_int4_sym_small(key, tokens):
    inp = small_inputs(key, tokens)
    w = inp.workload
    y = oracle.rht(inp.values, inp.signs, w.block)
    codes, scales = P.gpu_int4_sym(inp)
    P.check_int4_sym(codes, scales, y)
    deq = P.gpu_dequant(kq.KQ_FMT_INT4_SYM, codes, scales, None, None, w.tokens, w.dim)
    want = oracle.dequant_int4_sym(oracle.quant.int4_from_nibble(oracle.unpack_nibbles(codes)),
                                   scales)
    assert np.array_equal(deq.view(np.uint32), want.view(np.uint32))


def test_int4_asym_small():
    inp = small_inputs("c5", 37)
    w = inp.workload
    y = oracle.rht(inp.values, inp.signs, w.block)
    codes, scales, zeros = P.gpu_int4_asym(inp)
    P.check_int4_asym(codes, scales, zeros, y)
    deq = P.gpu_dequant(kq.KQ_FMT_INT4_ASYM, codes, scales, zeros, None, w.tokens, w.dim, 128)
    want = oracle.dequant_int4_asym(oracle.unpack_nibbles(codes), scales, zeros, 128)
    assert np.array_equal(deq.view(np.uint32), want.view(np.uint32))


def test_int4_asym_other_rotations():
    """Asymmetric g128 after a full-row rotation and with signs."""
    rng = np.random.default_rng(11)
    x = wl.round_to_bf16(rng.standard_normal((7, 4096)) * 3)
    s = (1 - 2 * rng.integers(0, 2, 4096)).astype(np.int8)
    for block in (0, 256):
        w = wl.Workload("x", 7, 4096, wl.BF16, block, True, wl.INT4_ASYM, 0, group=128)
        inp = P.inputs_from_values(w, x, s)
        c, sc, z = P.gpu_int4_asym(inp)
        P.check_int4_asym(c, sc, z, oracle.rht(x, s, block))


@pytest.mark.parametrize("dim,tokens,signs", [
    (4096, 43, True),             # tensor-core block kernel with sign flips
    (12288, 11, True),            # 96 column blocks per row
    (4096, 4 * 148 * 6 + 3, False),   # several tiles per CTA, overlapped last tile
    (4096, 3, True),              # 96 units: below one tile, general kernel
    (1024, 129, True),            # ragged: 1032 units
])
def test_int4_asym_block128_shapes(dim, tokens, signs):
    rng = np.random.default_rng(dim + tokens)
    x = rng.standard_normal((tokens, dim)) * np.exp(rng.standard_normal(dim))[None, :]
    x[:, rng.choice(dim, 4, replace=False)] *= 30
    edges = wl.edge_rows(dim, wl.BF16)[: max(0, min(6, tokens - 1))]
    x = wl.round_to_bf16(np.concatenate([x[: tokens - len(edges)], edges]))
    sg = (1 - 2 * rng.integers(0, 2, dim)).astype(np.int8) if signs else None
    w = wl.Workload("x", tokens, dim, wl.BF16, 128, signs, wl.INT4_ASYM, 0, group=128)
    inp = P.inputs_from_values(w, x, sg)
    c, sc, z = P.gpu_int4_asym(inp)
    P.check_int4_asym(c, sc, z, oracle.rht(x, sg, 128))


# --------------------------------------------------------------- NVFP4
@pytest.mark.parametrize("key,tokens", [("c2", 37), ("c4", 37), ("c2", 4 * 148 * 6 + 1),
                                        ("c2", 3)])
def test_nvfp4_small_dynamic_and_static(key, tokens):
    inp = small_inputs(key, tokens)
    w = inp.workload
    y = oracle.rht(inp.values, inp.signs, w.block)
    codes, bs, ts = P.gpu_nvfp4(inp)
    P.check_nvfp4(codes, bs, ts, y)
    # static mode with the same tensor scale gives identical output
    codes2, bs2, ts2 = P.gpu_nvfp4(inp, tensor_scale=ts)
    assert np.array_equal(codes2, codes) and np.array_equal(bs2, bs) and ts2 == ts
    # static mode with another tensor scale (saturating and subnormal scales)
    for f in (0.37, 4.0, 1e-3):
        t = np.float32(ts * f)
        c3, b3, _ = P.gpu_nvfp4(inp, tensor_scale=t)
        P.check_nvfp4(c3, b3, t, y, tensor_scale=t)
    deq = P.gpu_dequant(kq.KQ_FMT_NVFP4, codes, bs, None, ts, w.tokens, w.dim)
    want = oracle.dequant_nvfp4(oracle.unpack_nibbles(codes), bs, ts)
    assert np.array_equal(deq.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("dim,tokens", [(128, 37), (256, 41), (512, 3)])
def test_nvfp4_block128_ragged_lane_groups(dim, tokens):
    """Block-128 NVFP4 with a block count that is not a multiple of a warp's
    eight blocks (four lanes per block): the idle lanes of the last step write
    nothing and the active ones stay exact, in both tensor-scale modes."""
    w = wl.Workload("c2", tokens, dim, wl.BF16, 128, True, wl.NVFP4, 13)
    inp = wl.make_inputs(w)
    y = oracle.rht(inp.values, inp.signs, 128)
    codes, bs, ts = P.gpu_nvfp4(inp)
    P.check_nvfp4(codes, bs, ts, y)
    t = np.float32(ts * 0.5)
    c2, b2, _ = P.gpu_nvfp4(inp, tensor_scale=t)
    P.check_nvfp4(c2, b2, t, y, tensor_scale=t)


@pytest.mark.parametrize("tokens", [600, 5])
def test_nvfp4_block128_dynamic_tied_rows(tokens):
    """Dynamic tensor scale when every row ties for the maximum (one row
    repeated): all rows are candidates of the exact-maximum step, at 600 more
    than its candidate list holds."""
    w = wl.Workload("c2", tokens, 256, wl.BF16, 128, True, wl.NVFP4, 21)
    inp = wl.make_inputs(w)
    inp = wl.Inputs(w, np.repeat(inp.values[:1], tokens, axis=0),
                    np.repeat(inp.stored[:1], tokens, axis=0), inp.signs)
    y = oracle.rht(inp.values, inp.signs, 128)
    codes, bs, ts = P.gpu_nvfp4(inp)
    assert ts == oracle.nvfp4_tensor_scale(y)
    P.check_nvfp4(codes, bs, ts, y)


def test_nvfp4_block128_dynamic_after_input_write():
    """The dynamic block-128 call right after a kernel that rewrites its input
    on the same stream (no synchronisation between them): every call sees the
    new input.  Its quantisation pass reads inputs before it waits for the
    statistics pass, which itself starts only after the writer is done."""
    w = wl.Workload("c2", 300, 4096, wl.BF16, 128, True, wl.NVFP4, 31)
    a = wl.make_inputs(w)
    b = wl.make_inputs(wl.Workload("c2", 300, 4096, wl.BF16, 128, True, wl.NVFP4, 32))
    src = [torch.from_numpy(i.stored.view(np.int16)).cuda().view(torch.bfloat16) for i in (a, b)]
    want = []
    for i in (a, b):
        y = oracle.rht(i.values, a.signs, 128)
        want.append((y, oracle.nvfp4_tensor_scale(y)))
    x = torch.empty_like(src[0])
    s = torch.from_numpy(a.signs).cuda()
    c, bs, t, ws = kq.empty_nvfp4(w.tokens, w.dim, 128)
    outs = []
    for k in (0, 1, 0, 1):
        x.copy_(src[k])
        kq.kq_rht_quant_nvfp4(x, 128, s, c, bs, t, ws, dynamic=True)
        outs.append((k, c.clone(), bs.clone(), t.clone()))
    torch.cuda.synchronize()
    for k, cc, bb, tt in outs:
        y, ts = want[k]
        assert np.float32(tt.item()) == ts
        P.check_nvfp4(cc.cpu().numpy(), bb.cpu().numpy(), ts, y)


def test_nvfp4_block128_dynamic_many_rows():
    """Dynamic block-128 NVFP4 on more rows than the quantisation pass screens
    for the exact maximum itself (the exact step then runs as a launch of its
    own), and on exactly that many rows."""
    for tokens in (8193, 8192):
        w = wl.Workload("c2", tokens, 256, wl.BF16, 128, True, wl.NVFP4, 23)
        inp = wl.make_inputs(w)
        y = oracle.rht(inp.values, inp.signs, 128)
        codes, bs, ts = P.gpu_nvfp4(inp)
        assert ts == oracle.nvfp4_tensor_scale(y)
        P.check_nvfp4(codes, bs, ts, y)


@pytest.mark.parametrize("key,tokens", [("c2", 2500), ("c4", 2500)])
def test_nvfp4_dynamic_every_row_a_candidate(key, tokens):
    """Identical rows all reach the global lower bound, so the dynamic global
    step transforms every row (more rows than its CTAs: several candidate
    rows per CTA)."""
    base = small_inputs(key, 1, with_edges=False)
    w = base.workload
    vals = np.repeat(base.values, tokens, axis=0)
    inp = P.inputs_from_values(w, vals, base.signs)
    y = np.repeat(oracle.rht(base.values, base.signs, w.block), tokens, axis=0)
    codes, bs, ts = P.gpu_nvfp4(inp)
    P.check_nvfp4(codes, bs, ts, y)
    assert (codes == codes[:1]).all() and (bs == bs[:1]).all()


def test_nvfp4_round_trip_c4_small():
    inp = small_inputs("c4", 37)
    w = inp.workload
    codes, bs, ts = P.gpu_nvfp4(inp)
    deq = P.gpu_dequant(kq.KQ_FMT_NVFP4, codes, bs, None, ts, w.tokens, w.dim)
    winv = wl.Workload("inv", w.tokens, w.dim, wl.F32, w.block, True, w.fmt, 0)
    back = P.gpu_rht(wl.Inputs(winv, deq.astype(np.float64), deq, inp.signs), inverse=True)
    want = oracle.rht_inverse(deq.astype(np.float64), inp.signs, w.block)
    P.check_rotation(back, want)
    # ||x - x'|| = ||y - y_hat||: per element at most one scale unit (half a
    # grid gap, or the saturation error), and a block whose E4M3 scale flushes
    # to zero (r <= 2^-10) holds only values below 6 t 2^-10
    err = np.linalg.norm(back - inp.values, axis=1)
    unit = np.repeat(oracle.e4m3_decode(bs), 16, axis=1) * np.float64(ts)
    unit = np.where(unit > 0, unit, 6.0 * np.float64(ts) * 2.0 ** -10)
    assert np.all(err <= np.sqrt(np.sum(unit ** 2, axis=1)) * 1.0001 + 1e-30)


@pytest.mark.parametrize("key", ["c2", "c4"])
def test_nvfp4_all_zero_tensor(key):
    w = wl.WORKLOADS[key].with_tokens(5)
    vals = np.zeros((5, 4096))
    inp = P.inputs_from_values(w, vals, wl.make_inputs(w).signs)
    codes, bs, ts = P.gpu_nvfp4(inp)
    assert ts == 0 and not bs.any() and not codes.any()


def test_zero_tokens_is_noop():
    x = torch.empty((0, 4096), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, 4096), dtype=torch.float32, device="cuda")
    kq.kq_rht(x, 0, None, out)


def test_deterministic_bitwise():
    inp = small_inputs("c3", 9)
    a = P.gpu_int4_sym(inp)
    b = P.gpu_int4_sym(inp)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    inp2 = small_inputs("c4", 9)
    assert np.array_equal(P.gpu_rht(inp2), P.gpu_rht(inp2))


# ------------------------------------------------------------ full size
def _sample_rows(t, k, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(t, size=min(k, t), replace=False).tolist())
    rows |= {0, t - 1}
    return np.array(sorted(rows))


@pytest.mark.parametrize("key", ["c1", "c3", "c5"])
def test_full_size_per_token_formats(key):
    """Every row of the workload at its full size, in the launch the benchmark
    times, against the oracle (row chunks on the CPU)."""
    w = wl.WORKLOADS[key]
    inp = P.full_inputs(key)
    got = P.gpu_int4_sym(inp) if w.fmt == wl.INT4_SYM else P.gpu_int4_asym(inp, w.group)
    c = P.check_all_rows(f"full {key} {w.fmt}", inp, got)
    assert c.rows == w.tokens and c.scale_mismatch == 0 and c.bad == 0


@pytest.mark.parametrize("key", ["c2", "c4"])
def test_full_size_nvfp4(key):
    """Dynamic tensor scale: the global scale equals the oracle's, and every
    row's block scales and codes match under it."""
    w = wl.WORKLOADS[key]
    inp = P.full_inputs(key)
    codes, bs, ts = P.gpu_nvfp4(inp)
    t_ref = P.oracle_tensor_scale(inp)
    assert np.float32(ts).view(np.uint32) == t_ref.view(np.uint32)
    c = P.check_all_rows(f"full {key} nvfp4 dynamic", inp, (codes, bs, ts), tensor_scale=t_ref)
    assert c.rows == w.tokens and c.scale_mismatch == 0 and c.bad == 0
    if key == "c4":
        # round trip through the two calls (dequant, then the inverse rotation)
        deq = P.gpu_dequant(kq.KQ_FMT_NVFP4, codes, bs, None, ts, w.tokens, w.dim)
        winv = wl.Workload("inv", w.tokens, w.dim, wl.F32, w.block, True, w.fmt, 0)
        back = P.gpu_rht(wl.Inputs(winv, deq.astype(np.float64), deq, inp.signs),
                         inverse=True)
        for r0, r1 in P.row_chunks(w.tokens, w.dim):
            want = oracle.rht_inverse(deq[r0:r1].astype(np.float64), inp.signs, w.block)
            P.check_rotation(back[r0:r1], want)


def test_full_size_nvfp4_static_headline():
    """The call the benchmark's headline times: the 16384 x 4096 batch with a
    static tensor scale (the oracle's own), every row."""
    w = wl.WORKLOADS["c4"]
    inp = P.full_inputs("c4")
    t_ref = P.oracle_tensor_scale(inp)
    codes, bs, ts = P.gpu_nvfp4(inp, tensor_scale=t_ref)
    c = P.check_all_rows("full c4 nvfp4 static", inp, (codes, bs, ts), tensor_scale=t_ref)
    assert c.rows == w.tokens and c.scale_mismatch == 0 and c.bad == 0


# ------------------------------------------------ dequant + inverse rotation
def _rows_with_tail(t, k, seed):
    rows = _sample_rows(t, k, seed)
    return np.unique(np.concatenate([rows, np.arange(max(0, t - 5), t)]))


@pytest.mark.parametrize("key,tokens,signs_mode", [
    ("c4", 37, "aligned"),       # tensor-core kernel, ragged last tile
    ("c4", 37, "none"),
    ("c4", 37, "offset8"),       # general kernel
    ("c4", 4 * 148 * 6 + 3, "aligned"),   # several tiles per CTA: every stage wraps
    ("c2", 37, "aligned"),       # NVFP4 on block-128 rotation
    ("c1", 37, "aligned"),       # INT4 symmetric, full 4096
    ("c3", 13, "aligned"),       # INT4 symmetric, H12 x H1024
    ("c5", 37, "none"),          # asymmetric INT4 g128, per-head H128
])
def test_dequant_rht_inverse_random_codes(key, tokens, signs_mode):
    ci = wl.make_coded_inputs(wl.WORKLOADS[key], tokens=tokens)
    got = P.gpu_dequant_rht_inverse(ci, signs_mode)
    rows = _rows_with_tail(tokens, 40, 3) if tokens > 64 else np.arange(tokens)
    use = signs_mode != "none" and ci.signs is not None
    P.check_rotation(got[rows], P.oracle_dequant_rht_inverse(ci, rows, use_signs=use))


@pytest.mark.parametrize("key,tokens,signs_mode", [
    ("c4", 37, "aligned"), ("c4", 4 * 148 * 6 + 3, "aligned"), ("c4", 37, "offset8"),
    ("c5", 37, "none"),
])
def test_dequant_rht_inverse_bf16_out(key, tokens, signs_mode):
    ci = wl.make_coded_inputs(wl.WORKLOADS[key], tokens=tokens)
    got = P.gpu_dequant_rht_inverse(ci, signs_mode, out_dtype="bf16")
    rows = _rows_with_tail(tokens, 40, 4) if tokens > 64 else np.arange(tokens)
    use = signs_mode != "none" and ci.signs is not None
    P.check_rotation_bf16(got[rows], P.oracle_dequant_rht_inverse(ci, rows, use_signs=use))


def test_dequant_rht_inverse_round_trip_c4():
    """Codes and scales from the oracle's NVFP4 of real rows (edge rows
    included); the fused call must give the oracle's inverse of them, and x'
    must lie within the quantization error of x."""
    inp = small_inputs("c4", 37)
    w = inp.workload
    y = oracle.rht(inp.values, inp.signs, w.block)
    codes, bs, ts = oracle.nvfp4(y)
    ci = wl.CodedInputs(w.with_tokens(inp.values.shape[0]), oracle.pack_nibbles(codes), bs,
                        None, ts, inp.signs)
    got = P.gpu_dequant_rht_inverse(ci)
    want = P.oracle_dequant_rht_inverse(ci)
    P.check_rotation(got, want)
    err = np.linalg.norm(got - inp.values, axis=1)
    unit = np.repeat(oracle.e4m3_decode(bs), 16, axis=1) * np.float64(ts)
    unit = np.where(unit > 0, unit, 6.0 * np.float64(ts) * 2.0 ** -10)
    assert np.all(err <= np.sqrt(np.sum(unit ** 2, axis=1)) * 1.0001 + 1e-6)


def test_dequant_rht_inverse_zero_tokens():
    ci = wl.make_coded_inputs(wl.WORKLOADS["c4"], tokens=1)
    out = torch.empty((0, 4096), dtype=torch.float32, device="cuda")
    c = torch.empty((0, 2048), dtype=torch.uint8, device="cuda")
    s = torch.empty((0, 256), dtype=torch.uint8, device="cuda")
    t = torch.ones(1, dtype=torch.float32, device="cuda")
    kq.kq_dequant_rht_inverse(kq.KQ_FMT_NVFP4, c, s, None, t, 0, 4096, 0, 0,
                              torch.from_numpy(ci.signs).cuda(), out)


def test_full_size_dequant_rht_inverse_c4():
    """The benchmark's round-trip launch (16384 x 4096 NVFP4 -> fp32) on random
    codes: every row against the oracle, and against the two-call path
    (dequant, then the inverse rotation) within fp32 rounding."""
    w = wl.WORKLOADS["c4"]
    ci = wl.make_coded_inputs(w)
    got = P.gpu_dequant_rht_inverse(ci)
    for r0, r1 in P.row_chunks(w.tokens, w.dim):
        rows = np.arange(r0, r1)
        P.check_rotation(got[rows], P.oracle_dequant_rht_inverse(ci, rows))
    deq = P.gpu_dequant(kq.KQ_FMT_NVFP4, ci.codes, ci.scales, None, ci.tensor_scale,
                        w.tokens, w.dim)
    winv = wl.Workload("inv", w.tokens, w.dim, wl.F32, w.block, True, w.fmt, 0)
    two = P.gpu_rht(wl.Inputs(winv, deq.astype(np.float64), deq, ci.signs), inverse=True)
    P.check_rotation(got, two.astype(np.float64))


# ------------------------------------------------------------------ MXFP4
@pytest.mark.parametrize("key,tokens,block,dtype", [
    ("c4", 37, 0, None),          # full 4096 rotation, bf16
    ("c2", 37, 128, None),        # block-128 rotation
    ("c3", 9, 0, None),           # H12 x H1024
    ("c1", 37, 0, None),          # fp32 input
    ("c4", 11, 32, None),         # Hadamard block = MX block
])
def test_mxfp4_parity(key, tokens, block, dtype):
    inp = small_inputs(key, tokens)
    w0 = inp.workload
    w = wl.Workload(w0.key, w0.tokens, w0.dim, w0.dtype, block if block else w0.block,
                    w0.use_signs, wl.NVFP4, w0.seed)
    inp = P.inputs_from_values(w, inp.values, inp.signs)
    y = oracle.rht(inp.values, inp.signs, w.block)
    codes, scales = P.gpu_mxfp4(inp)
    P.check_mxfp4(codes, scales, y)
    deq = P.gpu_dequant(kq.KQ_FMT_MXFP4, codes, scales, None, None, w.tokens, w.dim)
    want = oracle.dequant_mxfp4(oracle.unpack_nibbles(codes), scales)
    assert np.array_equal(deq.view(np.uint32), want.view(np.uint32))


def test_mxfp4_round_trip_fused():
    inp = small_inputs("c4", 37)
    w = inp.workload
    y = oracle.rht(inp.values, inp.signs, w.block)
    codes, sc = oracle.mxfp4(y)
    ci = wl.CodedInputs(w.with_tokens(inp.values.shape[0]), oracle.pack_nibbles(codes), sc,
                        None, None, inp.signs)
    wmx = wl.Workload(w.key, ci.workload.tokens, w.dim, w.dtype, w.block, True, "mxfp4", 0)
    ci = wl.CodedInputs(wmx, ci.codes, ci.scales, None, None, inp.signs)
    got = P.gpu_dequant_rht_inverse(ci)
    deq = oracle.dequant_mxfp4(codes, sc).astype(np.float64)
    P.check_rotation(got, oracle.rht_inverse(deq, inp.signs, w.block))


def test_full_size_mxfp4_c4():
    w = wl.WORKLOADS["c4"]
    inp = P.full_inputs("c4")
    codes, scales = P.gpu_mxfp4(inp)
    total = P.Counts()
    for r0, r1 in P.row_chunks(w.tokens, w.dim):
        y = oracle.rht(inp.values[r0:r1], inp.signs, w.block)
        total = total + P.check_mxfp4(codes[r0:r1], scales[r0:r1], y, name=False)
    P.record("full c4 mxfp4", total)
    assert total.rows == w.tokens


# -------------------------------------------------------- KV-cache writer
@pytest.mark.parametrize("tokens,num_slots", [(43, 64), (3, 8), (4 * 148 * 6 + 3, 4000)])
def test_kv_cache_writer(tokens, num_slots):
    """Asymmetric INT4 g128 of per-head H_128 rotations, written to the cache
    rows a slot mapping names: named rows hold the oracle's result, the rest
    keep their previous contents."""
    w = wl.WORKLOADS["c5"].with_tokens(tokens)
    inp = wl.make_inputs(w)
    rng = np.random.default_rng(tokens)
    slots = rng.permutation(num_slots)[:tokens].astype(np.int64) if tokens <= num_slots \
        else rng.integers(0, num_slots, tokens)
    slots[rng.random(tokens) < 0.1] = -1                 # padding
    slots[rng.random(tokens) < 0.05] = num_slots + 3     # out of range: skipped
    dev = "cuda"
    x = torch.from_numpy(inp.stored.view(np.int16)).to(dev).view(torch.bfloat16)
    sm = torch.from_numpy(slots).to(dev)
    cc = torch.full((num_slots, w.dim // 2), 0xAB, dtype=torch.uint8, device=dev)
    sc = torch.full((num_slots, w.dim // 128), 7.0, dtype=torch.float16, device=dev)
    zc = torch.full((num_slots, w.dim // 128), -3.0, dtype=torch.float16, device=dev)
    kq.kq_rht_quant_int4_kv(x, None, sm, cc, sc, zc)
    torch.cuda.synchronize()
    cc, sc, zc = cc.cpu().numpy(), sc.cpu().numpy(), zc.cpu().numpy()
    ok = (slots >= 0) & (slots < num_slots)
    y = oracle.rht(inp.values[ok], None, 128)
    P.check_int4_asym(cc[slots[ok]], sc[slots[ok]], zc[slots[ok]], y)
    untouched = np.setdiff1d(np.arange(num_slots), slots[ok])
    assert np.all(cc[untouched] == 0xAB)
    assert np.all(sc[untouched] == 7.0) and np.all(zc[untouched] == -3.0)
