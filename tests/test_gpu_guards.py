"""Guard bytes: every output of every entry point sits between two 4 KB
margins filled with a known byte, and after the call the margins must be
intact -- no kernel writes outside its output tensors.  The token counts are
ragged on purpose: partial four-token tiles of the 4096-wide tensor-core
kernels (forward and inverse), the overlapped last tile of the block-128 GEMM
kernel, TMA boxes that reach past the end of the input, tails of the
warp-per-row and row-per-CTA kernels.  Each guarded result must also equal
the same call on plain tensors."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from hadamard_rotated_activation_b200 import workloads as wl
import hadamard_rotated_activation_b200 as kq

pytestmark = pytest.mark.gpu

MARGIN = 4096
FILL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


class Guarded:
    """Output tensors carved out of buffers with guard margins on both sides."""

    def __init__(self):
        self.bufs = []

    def __call__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        buf = torch.full((n + 2 * MARGIN,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, n))
        return buf[MARGIN:MARGIN + n].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        for i, (buf, n) in enumerate(self.bufs):
            head, tail = buf[:MARGIN], buf[MARGIN + n:]
            assert bool((head == FILL).all()), f"{what}: write before output {i}"
            assert bool((tail == FILL).all()), f"{what}: write after output {i}"


def _input(dim, tokens, dtype=wl.BF16, block=0, seed=0, signs=True):
    w = wl.Workload("c4", tokens, dim, dtype, block, signs, wl.NVFP4, seed)
    inp = wl.make_inputs(w)
    if dtype == wl.BF16:
        x = torch.from_numpy(inp.stored.view(np.int16)).cuda().view(torch.bfloat16)
    else:
        x = torch.from_numpy(inp.stored).cuda()
    s = torch.from_numpy(inp.signs).cuda() if inp.signs is not None else None
    return x, s


def _same(a, b, what):
    assert torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)), what


# (dim, block, dtype, tokens): which kernel each reaches is noted
ROT_SHAPES = [
    (4096, 0, wl.BF16, 37),      # 4096-wide tensor-core kernel, last tile holds one token
    (12288, 0, wl.BF16, 13),     # 12288-wide tensor-core kernel
    (4096, 128, wl.BF16, 37),    # block-128
    (2048, 0, wl.BF16, 37),      # warp per row
    (4096, 0, wl.F32, 37),       # fp32 input
    (384, 0, wl.BF16, 9),        # row per CTA, Paley 384
]


@pytest.mark.parametrize("dim,block,dtype,tokens", ROT_SHAPES)
def test_guards_rotation_and_int4_sym(dim, block, dtype, tokens):
    x, s = _input(dim, tokens, dtype, block)
    G = Guarded()
    out = G((tokens, dim), torch.float32)
    kq.kq_rht(x, block, s, out)
    G.check("kq_rht")
    ref = torch.empty((tokens, dim), dtype=torch.float32, device="cuda")
    kq.kq_rht(x, block, s, ref)
    _same(out, ref, "kq_rht")
    G = Guarded()
    codes, scales = G((tokens, dim // 2), torch.uint8), G((tokens,), torch.float32)
    kq.kq_rht_quant_int4(x, block, s, 0, False, codes, scales)
    G.check("kq_rht_quant_int4 sym")
    c2, s2 = kq.empty_int4_sym(tokens, dim)
    kq.kq_rht_quant_int4(x, block, s, 0, False, c2, s2)
    _same(codes, c2, "codes")
    _same(scales, s2, "scales")


@pytest.mark.parametrize("dim,tokens,signs", [
    (4096, 37, False),           # block-128 GEMM kernel: 1184 units, overlapped last tile
    (4096, 4 * 148 + 5, True),   # several tiles per CTA
    (4096, 3, True),             # below one tile: general kernel
    (12288, 5, True),
])
def test_guards_int4_asym(dim, tokens, signs):
    x, s = _input(dim, tokens, block=128, signs=signs)
    G = Guarded()
    codes = G((tokens, dim // 2), torch.uint8)
    scales = G((tokens, dim // 128), torch.float16)
    zeros = G((tokens, dim // 128), torch.float16)
    kq.kq_rht_quant_int4(x, 128, s, 128, True, codes, scales, zeros)
    G.check("kq_rht_quant_int4 asym")
    c2, s2, z2 = kq.empty_int4_asym(tokens, dim, 128)
    kq.kq_rht_quant_int4(x, 128, s, 128, True, c2, s2, z2)
    for a, b in ((codes, c2), (scales, s2), (zeros, z2)):
        _same(a, b, "asym")


NV_SHAPES = [
    (4096, 0, 37),               # 4096-wide tensor-core kernel (statistics pass too)
    (4096, 128, 37),             # block-128 kernel, four lanes per block
    (128, 128, 37),              # the same with a ragged last step (37 blocks)
    (2048, 0, 37),               # warp per row
    (12288, 0, 7),               # row per CTA
]


@pytest.mark.parametrize("dim,block,tokens", NV_SHAPES)
@pytest.mark.parametrize("dynamic", [False, True])
def test_guards_nvfp4(dim, block, tokens, dynamic):
    x, s = _input(dim, tokens, block=block)
    c2, b2, t2, ws2 = kq.empty_nvfp4(tokens, dim, block)
    kq.kq_rht_quant_nvfp4(x, block, s, c2, b2, t2, ws2, dynamic=True)
    torch.cuda.synchronize()
    G = Guarded()
    codes = G((tokens, dim // 2), torch.uint8)
    bs = G((tokens, dim // 16), torch.uint8)
    ts = G((1,), torch.float32)
    ws = G((ws2.numel(),), torch.uint8) if dynamic else None
    if not dynamic:
        ts.copy_(t2)
    kq.kq_rht_quant_nvfp4(x, block, s, codes, bs, ts, ws, dynamic=dynamic)
    G.check(f"kq_rht_quant_nvfp4 {'dynamic' if dynamic else 'static'}")
    for a, b in ((codes, c2), (bs, b2), (ts, t2)):
        _same(a, b, "nvfp4")


@pytest.mark.parametrize("dim,block,tokens", [(4096, 0, 37), (4096, 128, 37), (12288, 0, 5)])
def test_guards_mxfp4(dim, block, tokens):
    x, s = _input(dim, tokens, block=block)
    G = Guarded()
    codes, scales = G((tokens, dim // 2), torch.uint8), G((tokens, dim // 32), torch.uint8)
    kq.kq_rht_quant_mxfp4(x, block, s, codes, scales)
    G.check("kq_rht_quant_mxfp4")
    c2, s2 = kq.empty_mxfp4(tokens, dim)
    kq.kq_rht_quant_mxfp4(x, block, s, c2, s2)
    _same(codes, c2, "mxfp4 codes")
    _same(scales, s2, "mxfp4 scales")


@pytest.mark.parametrize("key,tokens", [("c4", 37), ("c4", 4 * 148 + 3), ("c5", 37),
                                        ("c1", 37), ("c2", 37)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_guards_dequant_and_inverse(key, tokens, out_dtype):
    ci = wl.make_coded_inputs(wl.WORKLOADS[key], tokens=tokens)
    w = ci.workload
    dev = "cuda"
    c = torch.from_numpy(np.ascontiguousarray(ci.codes)).to(dev)
    sc = torch.from_numpy(np.ascontiguousarray(ci.scales)).to(dev)
    z = None if ci.zeros is None else torch.from_numpy(np.ascontiguousarray(ci.zeros)).to(dev)
    t = None if ci.tensor_scale is None else torch.tensor([float(ci.tensor_scale)],
                                                          dtype=torch.float32, device=dev)
    sg = None if ci.signs is None else torch.from_numpy(ci.signs).to(dev)
    fmt = {wl.INT4_SYM: kq.KQ_FMT_INT4_SYM, wl.INT4_ASYM: kq.KQ_FMT_INT4_ASYM,
           wl.NVFP4: kq.KQ_FMT_NVFP4}[w.fmt]
    G = Guarded()
    out = G((tokens, w.dim), out_dtype)
    kq.kq_dequant_rht_inverse(fmt, c, sc, z, t, tokens, w.dim, w.block, w.group, sg, out)
    G.check("kq_dequant_rht_inverse")
    ref = torch.empty((tokens, w.dim), dtype=out_dtype, device=dev)
    kq.kq_dequant_rht_inverse(fmt, c, sc, z, t, tokens, w.dim, w.block, w.group, sg, ref)
    _same(out, ref, "dequant + inverse")
    if out_dtype == torch.float32:
        G = Guarded()
        d = G((tokens, w.dim), torch.float32)
        kq.kq_dequant(fmt, c, sc, z, t, tokens, w.dim, w.group, d)
        G.check("kq_dequant")


def test_guards_kv_cache_writer():
    tokens, slots_n = 4 * 148 + 5, 1000
    w = wl.WORKLOADS["c5"].with_tokens(tokens)
    inp = wl.make_inputs(w)
    x = torch.from_numpy(inp.stored.view(np.int16)).cuda().view(torch.bfloat16)
    rng = np.random.default_rng(5)
    slots = rng.permutation(slots_n)[:tokens].astype(np.int64)
    slots[:4] = [0, slots_n - 1, -1, slots_n + 7]       # both ends, padding, out of range
    sm = torch.from_numpy(slots).cuda()
    G = Guarded()
    cc = G((slots_n, w.dim // 2), torch.uint8)
    sc = G((slots_n, w.dim // 128), torch.float16)
    zc = G((slots_n, w.dim // 128), torch.float16)
    kq.kq_rht_quant_int4_kv(x, None, sm, cc, sc, zc)
    G.check("kq_rht_quant_int4_kv")
