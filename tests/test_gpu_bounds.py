"""GPU: the tensor-core rotations stay inside the error bounds that their
exact-scale screens assume, on adversarial bf16 rows, and the exact scales
hold on those rows.

A candidate screen keeps every output within 2E of the fp32 maximum, with E
the kernel's bound on |S_hat - S|; a bound that failed on some input range
would let the screen miss the true maximum and the scale would be wrong with
no other symptom.  The rows here stress what the tensor-core accumulation
model covers: exponents spread over 80 binades, a few huge values among tiny
ones, bf16 subnormals next to normal values, mantissas of all ones, heavy
cancellation, values in one binade.

Bounds (S = the unnormalized transform of the sign-flipped row):
  * 4096 wide (H_128 on the tensor cores, H_32 in registers):
    2.5 u W + 5 u (1 + 5 u) sum|x| + R with W <= 8 sum|x| and R <= 4 u sum|x|,
    so at most 30 u sum|x|;
  * 12288 wide (H_128 on the tensor cores, H_8 and the Paley H_12 in
    registers): 103 u sum|x|.
kq_rht writes fl(S_hat * fl(1/sqrt(n))), which adds at most 2 u |y| to the
bound scaled by 1/sqrt(n) (u = 2^-24).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from hadamard_rotated_activation_b200 import workloads as wl
import hadamard_rotated_activation_b200 as kq
import parity as P

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kq.lib()


def _bf16_from(sign, exp, mant):
    """sign * 2^exp * (1 + mant/128), exactly representable in bf16."""
    return sign * np.ldexp(1.0 + mant / 128.0, exp)


def adversarial_rows(dim: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = []
    sgn = lambda: rng.choice([-1.0, 1.0], dim)
    # exponents spread over 80 binades
    rows.append(_bf16_from(sgn(), rng.integers(-40, 41, dim), rng.integers(0, 128, dim)))
    # tiny values with a few huge ones
    r = _bf16_from(sgn(), rng.integers(-24, -18, dim), rng.integers(0, 128, dim))
    r[rng.choice(dim, 16, replace=False)] = _bf16_from(sgn()[:16], 13, rng.integers(0, 128, 16))
    rows.append(r)
    # bf16 subnormals (m 2^-133) next to values near one
    r = sgn() * rng.integers(1, 128, dim) * 2.0 ** -133
    r[::7] = _bf16_from(sgn()[::7], 0, rng.integers(0, 128, len(r[::7])))
    rows.append(r)
    # mantissas of all ones over eleven binades
    rows.append(_bf16_from(sgn(), rng.integers(-5, 6, dim), np.full(dim, 127)))
    # heavy cancellation: one magnitude, random signs
    rows.append(sgn() * 1.0)
    # one binade
    rows.append(_bf16_from(sgn(), np.zeros(dim, dtype=np.int64), rng.integers(0, 128, dim)))
    # pairs that cancel exactly except for a tiny residue
    r = _bf16_from(sgn(), rng.integers(0, 4, dim), rng.integers(0, 128, dim))
    r[1::2] = -r[0::2]
    r[5] = 2.0 ** -30
    rows.append(r)
    x = np.stack(rows)
    assert np.array_equal(_bits(x).astype(np.uint32) << 16, x.astype(np.float32).view(np.uint32)), \
        "every value is a bf16"
    return x


def _bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of values that bf16 holds exactly (subnormals included:
    a bf16 is the upper half of the fp32 of the same value)."""
    f = x.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), x)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def _inputs(w, x, signs):
    return wl.Inputs(w.with_tokens(x.shape[0]), x, _bits(x), signs)


@pytest.mark.parametrize("dim,coef", [(4096, 30.0), (12288, 103.0)])
@pytest.mark.parametrize("signed", [False, True])
def test_rotation_within_screen_bound(dim, coef, signed):
    x = adversarial_rows(dim, seed=dim + signed)
    rng = np.random.default_rng(5)
    signs = (1 - 2 * rng.integers(0, 2, dim)).astype(np.int8) if signed else None
    w = wl.Workload("c4" if dim == 4096 else "c3", x.shape[0], dim, wl.BF16, 0, signed,
                    wl.NVFP4 if dim == 4096 else wl.INT4_SYM, 0)
    inp = _inputs(w, x, signs)
    y = P.gpu_rht(inp)
    y_ref = oracle.rht(x, signs, 0)
    bound = coef * U * np.abs(x).sum(axis=1, keepdims=True) / np.sqrt(dim) * (1 + 2.0 ** -20) \
        + 2 * U * np.abs(y_ref)
    err = np.abs(y.astype(np.float64) - y_ref)
    worst = (err / bound).max()
    assert np.all(err <= bound), f"bound exceeded: worst {worst:.3g} x bound"


def test_exact_scales_on_adversarial_rows_12288():
    """Per-token INT4 on the adversarial rows: scales bit for bit."""
    x = adversarial_rows(12288, seed=77)
    rng = np.random.default_rng(6)
    signs = (1 - 2 * rng.integers(0, 2, 12288)).astype(np.int8)
    w = wl.Workload("c3", x.shape[0], 12288, wl.BF16, 0, True, wl.INT4_SYM, 0)
    inp = _inputs(w, x, signs)
    codes, scales = P.gpu_int4_sym(inp)
    P.check_int4_sym(codes, scales, oracle.rht(x, signs, 0))


def test_exact_scales_on_adversarial_rows_4096():
    """NVFP4 (dynamic and static tensor scale) on the adversarial rows: block
    scales and the tensor scale bit for bit."""
    x = adversarial_rows(4096, seed=78)
    x = np.concatenate([x] * 6)   # 42 rows: several 4-token tiles and a ragged one
    rng = np.random.default_rng(7)
    signs = (1 - 2 * rng.integers(0, 2, 4096)).astype(np.int8)
    w = wl.Workload("c4", x.shape[0], 4096, wl.BF16, 0, True, wl.NVFP4, 0)
    inp = _inputs(w, x, signs)
    xd, sd = P.to_device(inp)
    y = oracle.rht(x, signs, 0)
    c, b, t, ws = kq.empty_nvfp4(w.tokens, 4096, 0)
    kq.kq_rht_quant_nvfp4(xd, 0, sd, c, b, t, ws, dynamic=True)
    torch.cuda.synchronize()
    P.check_nvfp4(c.cpu().numpy(), b.cpu().numpy(), np.float32(t.item()), y)
    assert np.float32(t.item()) == oracle.nvfp4_tensor_scale(y)
    c2, b2, t2, _ = kq.empty_nvfp4(w.tokens, 4096, 0)
    t2.fill_(float(np.float32(t.item())) * 0.75)   # a static scale that saturates some blocks
    kq.kq_rht_quant_nvfp4(xd, 0, sd, c2, b2, t2, None, dynamic=False)
    torch.cuda.synchronize()
    ts = np.float32(t2.item())
    P.check_nvfp4(c2.cpu().numpy(), b2.cpu().numpy(), ts, y, tensor_scale=ts)
