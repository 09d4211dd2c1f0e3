"""CPU oracle for the randomized Hadamard rotation + 4-bit quantization path.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py` may import this package.  The product path (the
CUDA library and its Python binding) never calls it and shares no code with it.

What it computes, in plain fp64 numpy:
  * Hadamard matrices from their textbook constructions (Sylvester, natural
    order; Paley construction I with q = 11; Kronecker products) --
    `hadamard.py`.
  * The rotation y = x . D . H^T / sqrt(b) per block of b columns, as a dense
    matrix product -- `rht.py`.
  * Scalar quantizers to per-token symmetric INT4, asymmetric INT4 with
    fp16 scale and zero-point per group, and NVFP4 (E2M1 codes, E4M3 scale per
    16 elements, fp32 tensor scale), plus their dequantizers -- `quant.py`.
  * The number formats E2M1, E4M3 and fp16 written from their public
    definitions -- `formats.py`.
  * The 4-bit GEMM that consumes NVFP4 activations and weights, C = A_hat .
    B_hat^T in float64, and the tensor-core scale-factor layout of the block
    scales -- `gemm.py` (imported as `oracle.gemm`).

Every function cites the passage of the source pages it follows.  Readings of
points the pages leave open are listed in the module docstrings.

Pins: every function here is checked by `tests/test_oracle_*.py` against
closed forms, brute force on tiny inputs, invariants (orthogonality, norm
preservation, exact inverse, half-step bounds) and exhaustive format tables.
"""

from . import gemm  # noqa: F401
from .hadamard import hadamard, paley12, sylvester, quadratic_residues  # noqa: F401
from .rht import rht, rht_inverse, rht_unnormalized  # noqa: F401
from .formats import (  # noqa: F401
    E2M1_GRID, e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, fp16_round,
)
from .quant import (  # noqa: F401
    int4_sym_per_token, int4_asym_group, nvfp4, nvfp4_tensor_scale,
    dequant_int4_sym, dequant_int4_asym, dequant_nvfp4, pack_nibbles,
    unpack_nibbles, mxfp4, mxfp4_exponents, dequant_mxfp4,
)
