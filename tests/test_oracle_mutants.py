"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a dropped
term, a wrong index, a flipped comparison), builds it, and runs the pin suite
against that build; the suite has to fail.  An unmodified copy built the same
way has to pass, so a failure means the mistake was seen and not that the
harness is broken.  Everything here runs on the CPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "s4r_oracle.c")
HDR = os.path.join(ROOT, "oracle", "s4r_oracle.h")

# (name, text in the source, replacement).  Each text occurs exactly once.
MUTANTS = [
    ("logit scale dropped", "z[row * L + i] = acc * inv_sqrt_r;", "z[row * L + i] = acc;"),
    ("logit scale 1/r", "const double inv_sqrt_r = 1.0 / sqrt((double)r);",
     "const double inv_sqrt_r = 1.0 / (double)r;"),
    ("encode basis transposed", "acc += S[t * d + e] * B[(int64_t)e * r + j];",
     "acc += S[t * d + e] * B[(int64_t)(j * d + e) % ((int64_t)d * r)];"),
    ("reconstruct basis transposed", "acc += C[t * r + j] * B[(int64_t)e * r + j];",
     "acc += C[t * r + j] * B[(int64_t)(j * d + e) % ((int64_t)d * r)];"),
    ("softmax max not subtracted in the aggregate",
     "acc += exp(z[row * L + i] - row_max[row]) / row_sum[row];", "acc += exp(z[row * L + i]) / row_sum[row];"),
    ("row normaliser dropped", "acc += exp(z[row * L + i] - row_max[row]) / row_sum[row];",
     "acc += exp(z[row * L + i] - row_max[row]);"),
    ("ties go to the higher position", "return (x->i < y->i) ? -1 : (x->i > y->i);",
     "return (x->i > y->i) ? -1 : (x->i < y->i);"),
    ("window one row short", "for (int64_t i = L - p->local_window; i < L; ++i)",
     "for (int64_t i = L - p->local_window + 1; i < L; ++i)"),
    ("window counted as candidates", "const int64_t c = p->n_coeff - p->local_window;",
     "const int64_t c = p->n_coeff;"),
    ("positions without the sink offset", "idx[e] = (int32_t)(all[e].i + p->n_sink);", "idx[e] = (int32_t)(all[e].i);"),
    ("GQA groups interleaved", "    const int32_t g = h / G;\n    const double *q",
     "    const int32_t g = h % Hkv;\n    const double *q"),
    ("concat rows take the wrong heads", "p->q[((int64_t)w * Hq + (g * G + j)) * dh + t];",
     "p->q[((int64_t)w * Hq + (j * Hkv + g) % Hq) * dh + t];"),
    ("attention scale dropped", "const double scale = 1.0 / sqrt((double)dh);", "const double scale = 1.0;"),
    ("sinks left out of attention", "const int64_t n_keys = s + n_sel;", "const int64_t n_keys = n_sel;"),
    ("attention uses the oldest window slot", "const double *q = p->q + ((int64_t)(W - 1) * Hq + h) * dh;",
     "const double *q = p->q + ((int64_t)0 * Hq + h) * dh;"),
    ("pool window one wider", "const int64_t half = pool_kernel / 2;", "const int64_t half = pool_kernel / 2 + 1;"),
    ("average pool counts the padding", "sum / (double)count;", "sum / (double)pool_kernel;"),
    ("average pool takes the maximum", "(pool_mode == S4R_ORACLE_POOL_MAX) ? m : sum / (double)count;",
     "m;"),
    ("average pool leaves out the right neighbours", "for (int64_t j = i - half; j <= i + half; ++j)",
     "for (int64_t j = i - half; j <= i + (pool_mode == S4R_ORACLE_POOL_MAX ? half : 0); ++j)"),
    ("per-head rows use group 0's basis slice",
     "acc += p->q[((int64_t)w * Hq + h) * dh + t] * p->basis_k[(int64_t)(g * dh + t) * r + k];",
     "acc += p->q[((int64_t)w * Hq + h) * dh + t] * p->basis_k[(int64_t)(t) * r + k];"),
    ("value rows rebuilt with the key basis", "s4r_oracle_reconstruct(cv, n_sel, p->rank_v, p->basis_v, Dp, vh);",
     "s4r_oracle_reconstruct(cv, n_sel, p->rank_v, p->basis_k, Dp, vh);"),
]


def _build(tmp_path, text):
    d = tmp_path / "src"
    d.mkdir()
    (d / "s4r_oracle.c").write_text(text)
    (d / "s4r_oracle.h").write_text(open(HDR).read())
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-o", str(lib),
                    str(d / "s4r_oracle.c"), "-lm"], check=True)
    return str(lib)


def _run_pins(lib):
    env = dict(os.environ, S4R_ORACLE_LIB=lib, OMP_NUM_THREADS="4")
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                           "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_unmodified_copy_passes(tmp_path):
    res = _run_pins(_build(tmp_path, open(SRC).read()))
    assert res.returncode == 0, res.stdout[-2000:]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site of '{name}' not unique"
    res = _run_pins(_build(tmp_path, src.replace(old, new)))
    assert res.returncode == 1, f"pins did not catch: {name}\n{res.stdout[-2000:]}"


# The basis oracle (oracle/basis.py, NumPy): mistakes planted in a copy of the
# module, which tests/test_oracle_basis_pins.py then loads instead.
BASIS_SRC = os.path.join(ROOT, "oracle", "basis.py")
BASIS_MUTANTS = [
    ("3:7 instead of 7:3", "n_recent = (7 * n + 5) // 10", "n_recent = (3 * n + 5) // 10"),
    ("recent share rounded down", "n_recent = (7 * n + 5) // 10", "n_recent = (7 * n) // 10"),
    ("uniform rows reach into the sinks", "uniform = [n_sink + (j * span) // n_uniform",
     "uniform = [(j * (span + n_sink)) // n_uniform"),
    ("recent share one row short", "recent = list(range(L - n_recent, L))", "recent = list(range(L - n_recent, L - 1))"),
    ("normalisation dropped", "out[nz] = A[nz] / norms[nz, None]", "out[nz] = A[nz]"),
    ("normalised by the squared norm", "out[nz] = A[nz] / norms[nz, None]", "out[nz] = A[nz] / (norms[nz, None] ** 2)"),
    ("smallest singular directions kept", "B = sign_convention(vt[:rank].T)", "B = sign_convention(vt[-rank:].T)"),
    ("sample transposed (left singular vectors)", "_, s, vt = np.linalg.svd(A, full_matrices=False)",
     "_, s, vt = np.linalg.svd(A.T, full_matrices=False)"),
    ("no sign convention", "        if B[d, k] < 0:\n", "        if False:\n"),
]


def _run_basis_pins(path):
    env = dict(os.environ, S4R_BASIS_ORACLE=path)
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_basis_pins.py"),
                           "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_basis_unmodified_copy_passes(tmp_path):
    p = tmp_path / "basis.py"
    p.write_text(open(BASIS_SRC).read())
    res = _run_basis_pins(str(p))
    assert res.returncode == 0, res.stdout[-2000:]


@pytest.mark.parametrize("name,old,new", BASIS_MUTANTS, ids=[m[0] for m in BASIS_MUTANTS])
def test_basis_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(BASIS_SRC).read()
    assert src.count(old) == 1, f"mutation site of '{name}' not unique"
    p = tmp_path / "basis.py"
    p.write_text(src.replace(old, new))
    res = _run_basis_pins(str(p))
    assert res.returncode == 1, f"pins did not catch: {name}\n{res.stdout[-2000:]}"
