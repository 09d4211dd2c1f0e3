"""GPU: NVFP4 block scales in the tensor-core layout, and the NVFP4 GEMM that
consumes rotated, quantized activations, against the oracle.

Tolerance of the GEMM (fp32 output).  Every product E2M1 * E4M3 * E2M1 * E4M3
is exact; the tensor core accumulates in fp32.  Take one accumulation step
per 16-element block (the scale granularity) and let each step lose what the
tensor-core model of the bf16 kernels allows: its sum truncated to fp32
(2^-23 of the magnitudes so far) plus each of its 16 terms truncated to a grid
2^-25 below the step's largest magnitude, together under 2^-21 of the
magnitudes so far.  With K / 16 steps,
  |C - C_ref| <= (K / 16 + 2) 2^-21 |ta tb| sum_k |a b| + 2^-22 |C_ref|
(the last term: the fp32 products ta tb and acc * (ta tb)).  bf16 output adds
half a bf16 ulp.  A wrong scale byte or a misplaced 16-block moves an output
by about 1/(K/16) of sum_k |a b| or more: above this bound for K <= 2^14.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from oracle import gemm as ogemm
from hadamard_rotated_activation_b200 import workloads as wl
import hadamard_rotated_activation_b200 as kq
import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gemm_tolerance(k, absum, cref, bf16=False):
    tol = (k / 16 + 2) * 2.0 ** -21 * absum + 2.0 ** -22 * np.abs(cref)
    if bf16:
        mag = np.abs(cref) + tol
        tol = tol + np.where(mag > 0, np.ldexp(1.0, np.frexp(np.where(mag > 0, mag, 1))[1] - 9),
                             0.0)
    return tol


def check_gemm(c_gpu, codes_a, sa, ta, codes_b, sb, tb, bf16=False, name=None):
    """codes: unpacked E2M1 codes, scales: linear; returns max error / tolerance."""
    cref = ogemm.nvfp4_gemm(codes_a, sa, ta, codes_b, sb, tb)
    absum = ogemm.nvfp4_gemm_abs(codes_a, sa, ta, codes_b, sb, tb)
    tol = gemm_tolerance(codes_a.shape[1], absum, cref, bf16)
    err = np.abs(c_gpu.astype(np.float64) - cref)
    bad = err > tol
    assert not bad.any(), (f"{int(bad.sum())} outputs outside the tolerance; worst "
                           f"{(err / np.maximum(tol, 1e-300)).max():.3g} x tol")
    return float((err / np.maximum(tol, 1e-300)).max())


def run_gemm(codes_a, sa_lin, ta, codes_b, sb_lin, tb, out_dtype=torch.float32):
    """Upload packed codes and layout scales, run kq_gemm_nvfp4."""
    m, k = codes_a.shape
    n = codes_b.shape[0]
    a = _dev(oracle.pack_nibbles(codes_a))
    b = _dev(oracle.pack_nibbles(codes_b))
    sa = _dev(ogemm.sf_mma_layout(sa_lin))
    sb = _dev(ogemm.sf_mma_layout(sb_lin))
    tat = torch.tensor([float(ta)], dtype=torch.float32, device="cuda")
    tbt = torch.tensor([float(tb)], dtype=torch.float32, device="cuda")
    c = torch.empty((m, n), dtype=out_dtype, device="cuda")
    kq.kq_gemm_nvfp4(a, sa, tat, b, sb, tbt, c)
    torch.cuda.synchronize()
    return c.float().cpu().numpy()


def _random(rng, rows, k):
    codes = rng.integers(0, 16, size=(rows, k))
    scales = rng.integers(0, 0x7F, size=(rows, k // 16)).astype(np.uint8)
    return codes, scales


# ------------------------------------------------------ scale layout
@pytest.mark.parametrize("dim,block,tokens", [
    (4096, 0, 37),          # 4096-wide tensor-core kernel (fix-up path included)
    (4096, 0, 300),
    (4096, 128, 37),        # block-128 kernel
    (2048, 0, 150),         # warp per row
    (12288, 0, 5),          # row per CTA
])
def test_scales_in_mma_layout(dim, block, tokens):
    """Same codes, and the block scales at the layout's positions; the padding
    rows keep their contents."""
    w = wl.Workload("c4", tokens, dim, wl.BF16, block, True, wl.NVFP4, 3)
    inp = wl.make_inputs(w)
    x, s = P.to_device(inp)
    c1, b1, t1, ws = kq.empty_nvfp4(tokens, dim, block)
    kq.kq_rht_quant_nvfp4(x, block, s, c1, b1, t1, ws, dynamic=True)
    c2, b2, t2, _ = kq.empty_nvfp4(tokens, dim, block, mma_layout=True)
    t2.copy_(t1)
    kq.kq_rht_quant_nvfp4(x, block, s, c2, b2, t2, None, dynamic=False, mma_layout=True)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    want = ogemm.sf_mma_layout(b1.cpu().numpy())
    assert np.array_equal(b2.cpu().numpy(), want)


# ------------------------------------------------------------- GEMM
@pytest.mark.parametrize("m,n,k", [(1, 128, 256), (37, 128, 512), (128, 256, 256),
                                   (300, 256, 12288), (4 * 148 * 2 + 7, 384, 1024)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_random_codes(m, n, k, out_dtype):
    """Uniform codes and finite E4M3 scales (zero and subnormal included);
    ragged M, several N tiles, long K, more tiles than CTAs."""
    rng = np.random.default_rng(m * 7 + n + k)
    a, sa = _random(rng, m, k)
    b, sb = _random(rng, n, k)
    ta, tb = np.float32(rng.lognormal(-4, 1)), np.float32(rng.lognormal(-6, 1))
    c = run_gemm(a, sa, ta, b, sb, tb, out_dtype)
    check_gemm(c, a, sa, ta, b, sb, tb, bf16=out_dtype == torch.bfloat16)


def test_gemm_zero_and_one_hot():
    k = 512
    a = np.zeros((5, k), dtype=np.int64)
    sa = np.zeros((5, k // 16), dtype=np.uint8)
    a[2, 300] = 2                        # E2M1 1.0
    sa[2, 300 // 16] = 0x38              # E4M3 1.0
    rng = np.random.default_rng(9)
    b, sb = _random(rng, 128, k)
    c = run_gemm(a, sa, 1.0, b, sb, 0.5)
    assert not c[[0, 1, 3, 4]].any()
    want = oracle.e2m1_decode(b[:, 300]) * oracle.e4m3_decode(sb[:, 300 // 16]) * 0.5
    assert np.array_equal(c[2], want.astype(np.float32))


def test_gemm_of_rotated_activations_c4():
    """The consumer of the 16384 x 4096 batch: its rotated NVFP4 codes (static
    tensor scale, scales in the tensor-core layout) times a 4096 x 4096 weight
    rotated and quantized by the same call, every output against the oracle's
    GEMM of the same codes; and the product stays close to X W^T (the rotation
    cancels between the two operands)."""
    w = wl.WORKLOADS["c4"]
    inp = P.full_inputs("c4")
    x, s = P.to_device(inp)
    rng = np.random.default_rng(44)
    wt = wl.round_to_bf16(rng.standard_normal((4096, 4096)) / 64.0)
    wdev = torch.from_numpy(wl.bf16_bits(wt).view(np.int16)).cuda().view(torch.bfloat16)
    ops = []
    for src, rows in ((x, w.tokens), (wdev, 4096)):
        c0, b0, t0, ws = kq.empty_nvfp4(rows, 4096, 0)
        kq.kq_rht_quant_nvfp4(src, 0, s, c0, b0, t0, ws, dynamic=True)
        cm, bm, tm, _ = kq.empty_nvfp4(rows, 4096, 0, mma_layout=True)
        tm.copy_(t0)
        kq.kq_rht_quant_nvfp4(src, 0, s, cm, bm, tm, None, dynamic=False, mma_layout=True)
        ops.append((cm, bm, tm, b0))
    out = torch.empty((w.tokens, 4096), dtype=torch.float32, device="cuda")
    (ca, sa, ta, sal), (cb, sb, tb, sbl) = ops
    kq.kq_gemm_nvfp4(ca, sa, ta, cb, sb, tb, out)
    torch.cuda.synchronize()
    codes_b = oracle.unpack_nibbles(cb.cpu().numpy())
    sbl = sbl.cpu().numpy()
    ta_, tb_ = np.float32(ta.item()), np.float32(tb.item())
    got = out.cpu().numpy()
    worst = 0.0
    for r0, r1 in P.row_chunks(w.tokens, 4096, budget=1 << 24):
        codes_a = oracle.unpack_nibbles(ca[r0:r1].cpu().numpy())
        worst = max(worst, check_gemm(got[r0:r1], codes_a, sal[r0:r1].cpu().numpy(), ta_,
                                      codes_b, sbl, tb_))
    # computational invariance: the product of the quantized rotated operands
    # approximates X W^T (a loose sanity bound; the quantization error is the rest)
    rows = np.arange(0, w.tokens, 512)
    xw = inp.values[rows] @ wt.T
    rel = np.linalg.norm(got[rows] - xw) / np.linalg.norm(xw)
    assert rel < 0.2, rel
