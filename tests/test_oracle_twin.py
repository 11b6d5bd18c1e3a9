"""The C oracle against its NumPy twin (oracle/twin.py).

Two independent readings of the same definitions (Eq. 3; Eqs. 8-10; pooling;
Eqs. 13-15; Eqs. 16-18): one in plain C loops, one in whole-array NumPy.  On
small random problems they must agree to 1e-12 (relative to the largest
value), and on the same score vector they must pick the same positions,
including vectors built from heavy ties.  A slip in either one (a dropped
term, a transposed operand, a wrong row order, a tie broken the other way)
shows up here.
"""
import numpy as np
import pytest

import oracle
from oracle import twin

TOL = 1e-12


def _problem(rng, *, W, Hq, Hkv, dh, rk, rv, s, L, w, k, pool_kernel=1, pool_mode=0, row_mode=0):
    Dp = Hkv * dh
    return oracle.Problem(q=rng.standard_normal((W, Hq, dh)), coeff_k=rng.standard_normal((L, rk)),
                          coeff_v=rng.standard_normal((L, rv)), basis_k=rng.standard_normal((Dp, rk)) / np.sqrt(Dp),
                          basis_v=rng.standard_normal((Dp, rv)) / np.sqrt(Dp), sink_k=rng.standard_normal((s, Dp)),
                          sink_v=rng.standard_normal((s, Dp)), n_heads_kv=Hkv, local_window=w, top_k=k,
                          pool_kernel=pool_kernel, row_mode=row_mode, pool_mode=pool_mode)


CASES = [
    dict(W=4, Hq=8, Hkv=2, dh=16, rk=12, rv=20, s=4, L=300, w=32, k=40),
    dict(W=2, Hq=4, Hkv=4, dh=8, rk=8, rv=8, s=0, L=50, w=8, k=10),
    dict(W=3, Hq=6, Hkv=1, dh=8, rk=6, rv=6, s=2, L=100, w=16, k=30, pool_kernel=7),
    dict(W=3, Hq=6, Hkv=1, dh=8, rk=6, rv=6, s=2, L=100, w=16, k=30, pool_kernel=7, pool_mode=1),
    dict(W=2, Hq=8, Hkv=2, dh=16, rk=16, rv=16, s=4, L=200, w=32, k=20, row_mode=1),
    dict(W=1, Hq=2, Hkv=1, dh=4, rk=4, rv=4, s=1, L=5, w=8, k=3),            # cache shorter than the window
    dict(W=1, Hq=2, Hkv=1, dh=4, rk=4, rv=4, s=3, L=0, w=8, k=3),            # empty cache: sinks only
    dict(W=2, Hq=4, Hkv=2, dh=8, rk=8, rv=8, s=4, L=64, w=0, k=64),          # k covers every candidate
    dict(W=2, Hq=4, Hkv=2, dh=8, rk=8, rv=8, s=4, L=64, w=16, k=0),          # window only
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_twin_agrees_with_the_c_oracle(case):
    rng = np.random.default_rng(1000 + CASES.index(case))
    p = _problem(rng, **case)
    out_c, idx_c, sc_c = oracle.decode_step(p)
    out_t, idx_t, sc_t = twin.decode_step(p)
    assert sc_t.shape == sc_c.shape
    if sc_c.size:
        assert np.abs(sc_t - sc_c).max() <= TOL * max(1.0, np.abs(sc_c).max())
    # the same score vector gives the same positions
    assert np.array_equal(twin.select(p, sc_c), idx_c)
    assert np.array_equal(oracle.select(p, sc_t), idx_t)
    # attention over the same selection
    ref = np.abs(out_c).max() if out_c.size else 1.0
    assert np.abs(twin.decode_given_idx(p, idx_c) - out_c).max() <= TOL * max(1.0, ref)
    if np.array_equal(idx_t, idx_c):
        assert np.abs(out_t - out_c).max() <= TOL * max(1.0, ref)


def test_twin_encode_reconstruct_and_pool_agree():
    rng = np.random.default_rng(7)
    S, B = rng.standard_normal((37, 24)), rng.standard_normal((24, 10))
    C = oracle.encode(S, B)
    assert np.abs(twin.encode(S, B) - C).max() <= TOL * np.abs(C).max()
    R = oracle.reconstruct(C, B)
    assert np.abs(twin.reconstruct(C, B) - R).max() <= TOL * np.abs(R).max()
    s = rng.standard_normal(50)
    for kernel in (1, 3, 7, 63):
        for mode in (oracle.POOL_MAX, oracle.POOL_AVG):
            for n in (0, 1, 5, 50):
                a, b = oracle.pool(s, n, kernel, mode), twin.pool(s, n, kernel, mode)
                assert a.shape == b.shape and (n == 0 or np.abs(a - b).max() <= TOL)


@pytest.mark.parametrize("pool_kernel,pool_mode", [(1, 0), (7, 0), (7, 1)])
def test_tie_heavy_scores_select_the_same_positions(pool_kernel, pool_mode):
    rng = np.random.default_rng(3)
    p = _problem(rng, W=1, Hq=2, Hkv=1, dh=4, rk=4, rv=4, s=4, L=400, w=16, k=100,
                 pool_kernel=pool_kernel, pool_mode=pool_mode)
    for levels in (1, 2, 3, 17):
        sc = rng.integers(0, levels, size=400).astype(np.float64)    # exact ties everywhere
        assert np.array_equal(twin.select(p, sc), oracle.select(p, sc))
