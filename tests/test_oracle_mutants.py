"""Planted mistakes: each one, written into a copy of the oracle, must make at
least one of the oracle's pins fail.  This is what shows that the pins are
strong enough to catch a plausible slip anywhere in the oracle (a transposed
operand, a wrong sign, constant, divisor, rounding rule, index order or
factor order), and not only the oracle's agreement with itself.

Each mutant is one textual substitution in one oracle file; the pin tests
(`tests/test_oracle_*.py`) run in a child process on a scratch copy of the
oracle, the pins and the input generator.  An unmodified copy must pass
(the control).
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["test_oracle_hadamard.py", "test_oracle_rht.py", "test_oracle_quant.py",
        "test_oracle_formats.py", "test_oracle_gemm.py"]

# (name, oracle file, text, replacement)
MUTANTS = [
    ("transposed H in the forward rotation", "rht.py",
     "s = xs.reshape(t * (n // b), b) @ h.T", "s = xs.reshape(t * (n // b), b) @ h"),
    ("sign vector dropped", "rht.py", "return x * s[None, :]", "return x"),
    ("wrong normalisation 1/b", "rht.py",
     "return rht_unnormalized(x, signs, block) / np.sqrt(np.float64(b))",
     "return rht_unnormalized(x, signs, block) / np.float64(b)"),
    ("wrong Paley sign (first column +1)", "hadamard.py", "s[1:, 0] = -1.0", "s[1:, 0] = 1.0"),
    ("swapped Kronecker factors", "hadamard.py",
     "h = np.kron(paley12(), sylvester(n // 12))", "h = np.kron(sylvester(n // 12), paley12())"),
    ("wrong INT4 divisor (8)", "quant.py", "scale = (amax / 7.0)", "scale = (amax / 8.0)"),
    ("wrong NVFP4 constant (E4M3 max 480)", "quant.py", "E4M3_MAX = 448.0", "E4M3_MAX = 480.0"),
    ("asymmetric zero-point sign", "quant.py", "np.rint(-mn / s64)", "np.rint(mn / s64)"),
    ("nibble order swapped", "quant.py",
     "(c[..., 0::2] | (c[..., 1::2] << 4))", "(c[..., 1::2] | (c[..., 0::2] << 4))"),
    ("MXFP4 exponent off by one", "quant.py",
     "e = ex.astype(np.int64) - 1 - E2M1_EMAX", "e = ex.astype(np.int64) - E2M1_EMAX"),
    ("E2M1 ties to odd", "formats.py",
     "even = tie & ((np.arange(8) & 1) == 0)[None, :]",
     "even = tie & ((np.arange(8) & 1) == 1)[None, :]"),
    ("E4M3 exponent bias 8", "formats.py",
     "mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)", "mag = (1.0 + m / 8.0) * 2.0 ** (e - 8)"),
    ("GEMM without the B tensor scale", "gemm.py",
     "* (np.float64(np.float32(ta)) * np.float64(np.float32(tb)))", "* np.float64(np.float32(ta))"),
    ("scale layout with row groups and lanes swapped", "gemm.py",
     "np.ascontiguousarray(t.transpose(0, 3, 2, 1, 4)).reshape(-1)",
     "np.ascontiguousarray(t.transpose(0, 3, 1, 2, 4)).reshape(-1)"),
]


def _scratch(dst):
    """oracle/, the pin tests (+ conftest and golden files) and the input
    generator, copied under dst."""
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    for f in PINS + ["conftest.py"]:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    pkg = os.path.join(dst, "hadamard_rotated_activation_b200")
    os.makedirs(pkg)
    open(os.path.join(pkg, "__init__.py"), "w").close()
    shutil.copy(os.path.join(ROOT, "hadamard_rotated_activation_b200", "workloads.py"), pkg)


def _start(dst):
    env = dict(os.environ)
    env.pop("PYTHONPATH", None)
    for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        env[v] = "1"
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "-m", "not gpu"] + [os.path.join("tests", f) for f in PINS]
    return subprocess.Popen(cmd, cwd=dst, env=env, stdout=subprocess.PIPE,
                            stderr=subprocess.STDOUT, text=True)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    procs = {}
    control = tmp_path / "control"
    _scratch(str(control))
    procs["control"] = _start(str(control))
    for i, (name, fname, old, new) in enumerate(MUTANTS):
        d = tmp_path / f"m{i}"
        _scratch(str(d))
        path = d / "oracle" / fname
        src = path.read_text()
        assert src.count(old) == 1, f"mutation site not unique or missing: {name}"
        path.write_text(src.replace(old, new))
        procs[name] = _start(str(d))
    out = {k: p.communicate(timeout=600) for k, p in procs.items()}
    rc = {k: p.returncode for k, p in procs.items()}
    assert rc["control"] == 0, "the unmodified copy must pass its pins:\n" + out["control"][0]
    survivors = [k for k in rc if k != "control" and rc[k] != 1]
    assert not survivors, f"planted mistakes no pin caught (or that crashed): {survivors}"
