"""fp64 CPU oracle for S4R compressed-KV decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library (``libs4r.so`` and
its Python binding) never imports, links or calls it, and the two share no
code.  The arithmetic lives in ``s4r_oracle.c`` (plain C, float64); this module
only compiles it with gcc and marshals numpy arrays through ctypes.

Method source: "S^4R: Selective Sampling, Subspaces, and Sparse Reconstruction
for Compressed Long-Context KV Caching" (arXiv 2608.00528), review page.  Each
C function cites the equation it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s4r_oracle.c")
_HDR = os.path.join(_HERE, "s4r_oracle.h")
_LIB = os.path.join(_HERE, "_build", "libs4r_oracle.so")

ROWS_CONCAT = 0
ROWS_PER_HEAD = 1
POOL_MAX = 0
POOL_AVG = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP).  Returns the library path."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= newest:
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    # -ffp-contract=off keeps every product and sum a separate IEEE float64
    # operation, exactly as written.
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("n_heads_q", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("rank_k", ctypes.c_int32), ("rank_v", ctypes.c_int32),
        ("n_sink", ctypes.c_int32), ("local_window", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("query_window", ctypes.c_int32), ("pool_kernel", ctypes.c_int32),
        ("row_mode", ctypes.c_int32), ("pool_mode", ctypes.c_int32),
        ("n_coeff", ctypes.c_int64),
        ("q", ctypes.c_void_p), ("coeff_k", ctypes.c_void_p), ("coeff_v", ctypes.c_void_p),
        ("basis_k", ctypes.c_void_p), ("basis_v", ctypes.c_void_p),
        ("sink_k", ctypes.c_void_p), ("sink_v", ctypes.c_void_p),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        # S4R_ORACLE_LIB: load another build of this source instead (the
        # mutation test points it at copies with planted mistakes).
        lib = ctypes.CDLL(os.environ.get("S4R_ORACLE_LIB") or build())
        P = ctypes.POINTER(_Problem)
        dp = ctypes.c_void_p
        lib.s4r_oracle_encode.argtypes = [dp, ctypes.c_int64, ctypes.c_int32, dp, ctypes.c_int32, dp]
        lib.s4r_oracle_encode.restype = None
        lib.s4r_oracle_reconstruct.argtypes = [dp, ctypes.c_int64, ctypes.c_int32, dp, ctypes.c_int32, dp]
        lib.s4r_oracle_reconstruct.restype = None
        lib.s4r_oracle_scores.argtypes = [P, dp]
        lib.s4r_oracle_pool.argtypes = [dp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, dp]
        lib.s4r_oracle_select.argtypes = [P, dp, dp]
        lib.s4r_oracle_decode_given_idx.argtypes = [P, dp, ctypes.c_int64, dp]
        lib.s4r_oracle_decode_step.argtypes = [P, dp, dp, dp]
        lib.s4r_oracle_threads.argtypes = []
        lib.s4r_oracle_set_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads the oracle uses (set OMP_NUM_THREADS before loading)."""
    return int(_load().s4r_oracle_threads())


def set_threads(n: int) -> int:
    """Use n OpenMP threads from now on (results do not depend on n)."""
    return int(_load().s4r_oracle_set_threads(int(n)))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


@dataclass
class Problem:
    """One decode problem in float64.  Shapes:
    q [W][H_q][d_h], coeff_k [L_c][r_k], coeff_v [L_c][r_v], basis_k [D'][r_k],
    basis_v [D'][r_v], sink_k / sink_v [s][D']."""
    q: np.ndarray
    coeff_k: np.ndarray
    coeff_v: np.ndarray
    basis_k: np.ndarray
    basis_v: np.ndarray
    sink_k: np.ndarray
    sink_v: np.ndarray
    n_heads_kv: int
    local_window: int
    top_k: int
    pool_kernel: int = 1
    row_mode: int = ROWS_CONCAT
    pool_mode: int = POOL_MAX

    def __post_init__(self):
        for name in ("q", "coeff_k", "coeff_v", "basis_k", "basis_v", "sink_k", "sink_v"):
            setattr(self, name, _f64(getattr(self, name)))
        W, Hq, dh = self.q.shape
        self.query_window, self.n_heads_q, self.head_dim = W, Hq, dh
        Dp = self.n_heads_kv * dh
        L = self.coeff_k.shape[0]
        self.n_coeff = L
        self.rank_k = self.basis_k.shape[1]
        self.rank_v = self.basis_v.shape[1]
        self.n_sink = self.sink_k.shape[0]
        assert Hq % self.n_heads_kv == 0
        assert self.basis_k.shape == (Dp, self.rank_k) and self.basis_v.shape == (Dp, self.rank_v)
        assert self.coeff_k.shape == (L, self.rank_k) and self.coeff_v.shape == (L, self.rank_v)
        assert self.sink_k.shape == (self.n_sink, Dp) and self.sink_v.shape == (self.n_sink, Dp)

    def _c(self) -> _Problem:
        return _Problem(self.n_heads_q, self.n_heads_kv, self.head_dim, self.rank_k, self.rank_v,
                        self.n_sink, self.local_window, self.top_k, self.query_window,
                        self.pool_kernel, self.row_mode, self.pool_mode, self.n_coeff,
                        _ptr(self.q), _ptr(self.coeff_k), _ptr(self.coeff_v), _ptr(self.basis_k),
                        _ptr(self.basis_v), _ptr(self.sink_k), _ptr(self.sink_v))


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def encode(states, basis) -> np.ndarray:
    """C = S . B (Eq. 3) in float64."""
    S, B = _f64(states), _f64(basis)
    n, d = S.shape
    assert B.shape[0] == d
    C = np.empty((n, B.shape[1]), dtype=np.float64)
    _load().s4r_oracle_encode(_ptr(S), n, d, _ptr(B), B.shape[1], _ptr(C))
    return C


def reconstruct(coeffs, basis) -> np.ndarray:
    """Rebuilt rows C . B^T (Eq. 16) in float64."""
    C, B = _f64(coeffs), _f64(basis)
    n, r = C.shape
    assert B.shape[1] == r
    out = np.empty((n, B.shape[0]), dtype=np.float64)
    _load().s4r_oracle_reconstruct(_ptr(C), n, r, _ptr(B), B.shape[0], _ptr(out))
    return out


def scores(p: Problem) -> np.ndarray:
    """Latent relevance score of every coefficient row (Eqs. 8-10)."""
    out = np.zeros(max(p.n_coeff, 1), dtype=np.float64)
    c = p._c()
    _check(_load().s4r_oracle_scores(ctypes.byref(c), _ptr(out)), "scores")
    return out[: p.n_coeff]


def pool(score_vec, n_cand: int, kernel: int, mode: int = POOL_MAX) -> np.ndarray:
    """Pooled candidate scores: max or mean over the in-range neighbours."""
    s = _f64(score_vec)
    out = np.empty(max(n_cand, 1), dtype=np.float64)
    _check(_load().s4r_oracle_pool(_ptr(s), n_cand, kernel, mode, _ptr(out)), "pool")
    return out[:n_cand]


def select(p: Problem, score_vec) -> np.ndarray:
    """Top-k absolute positions, ascending, -1 padded (Eqs. 13-15)."""
    s = _f64(score_vec)
    idx = np.full(max(p.top_k, 1), -1, dtype=np.int32)
    c = p._c()
    _check(_load().s4r_oracle_select(ctypes.byref(c), _ptr(s), _ptr(idx)), "select")
    return idx[: p.top_k]


def decode_given_idx(p: Problem, idx) -> np.ndarray:
    """Attention output [H_q][d_h] over sinks + the given positions + the window."""
    ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    out = np.empty((p.n_heads_q, p.head_dim), dtype=np.float64)
    c = p._c()
    _check(_load().s4r_oracle_decode_given_idx(ctypes.byref(c), _ptr(ix), ix.size, _ptr(out)),
           "decode_given_idx")
    return out


def decode_step(p: Problem):
    """One decode step: returns (out [H_q][d_h], idx [top_k], scores [L_c])."""
    out = np.empty((p.n_heads_q, p.head_dim), dtype=np.float64)
    idx = np.full(max(p.top_k, 1), -1, dtype=np.int32)
    sc = np.zeros(max(p.n_coeff, 1), dtype=np.float64)
    c = p._c()
    _check(_load().s4r_oracle_decode_step(ctypes.byref(c), _ptr(out), _ptr(idx), _ptr(sc)),
           "decode_step")
    return out, idx[: p.top_k], sc[: p.n_coeff]
