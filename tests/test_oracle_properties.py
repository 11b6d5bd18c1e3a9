"""Randomised properties of the decode oracle (Hypothesis), on the CPU.

Over random small shapes (both row modes, both pooling modes, sinks or none,
caches shorter than the window, k above and below the candidates), the C
oracle and its NumPy twin must agree, and the C oracle must satisfy what the
definitions fix whatever the shape:
  * each row's softmax sums to 1, so the scores sum to the number of rows
    (W * G for CONCAT rows, W * H_q per head), Eqs. 8-10;
  * idx lists min(k, candidates) distinct positions s + i, i < L_c - w, in
    ascending order, -1 padded, and they are the top of a brute-force
    ranking (larger key first, lower position on ties), Eqs. 13-15;
  * each output column of a head lies between the smallest and the largest
    value it attends to (a softmax average), Eqs. 16-18.
"""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from oracle import twin


@st.composite
def problems(draw):
    Hkv = draw(st.sampled_from([1, 2, 4]))
    G = draw(st.sampled_from([1, 2, 4]))
    dh = draw(st.sampled_from([4, 8]))
    W = draw(st.integers(1, 4))
    rk, rv = draw(st.integers(1, 12)), draw(st.integers(1, 12))
    s = draw(st.integers(0, 4))
    L = draw(st.integers(0, 90))
    w = draw(st.integers(0, 20))
    k = draw(st.integers(0, 40))
    pool_kernel = draw(st.sampled_from([1, 3, 7]))
    pool_mode = draw(st.sampled_from([oracle.POOL_MAX, oracle.POOL_AVG]))
    row_mode = draw(st.sampled_from([oracle.ROWS_CONCAT, oracle.ROWS_PER_HEAD]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    Dp, Hq = Hkv * dh, Hkv * G
    return oracle.Problem(q=rng.standard_normal((W, Hq, dh)), coeff_k=rng.standard_normal((L, rk)),
                          coeff_v=rng.standard_normal((L, rv)), basis_k=rng.standard_normal((Dp, rk)),
                          basis_v=rng.standard_normal((Dp, rv)), sink_k=rng.standard_normal((s, Dp)),
                          sink_v=rng.standard_normal((s, Dp)), n_heads_kv=Hkv, local_window=w, top_k=k,
                          pool_kernel=pool_kernel, row_mode=row_mode, pool_mode=pool_mode)


@settings(max_examples=120, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(problems())
def test_oracle_properties_and_twin(p):
    out, idx, sc = oracle.decode_step(p)
    W, Hq, dh = p.q.shape
    G = Hq // p.n_heads_kv
    L, w, k, s = p.n_coeff, p.local_window, p.top_k, p.n_sink
    # scores: one unit of probability per row
    rows = W * (G if p.row_mode == oracle.ROWS_CONCAT else Hq)
    if L:
        assert abs(sc.sum() - rows) <= 1e-9 * rows
        assert (sc >= 0).all()
    # selection: well formed and the top of a brute-force ranking
    n_cand = max(L - w, 0)
    n_take = min(k, n_cand)
    assert idx.shape == (k,)
    assert (idx[n_take:] == -1).all()
    top = idx[:n_take]
    assert (np.diff(top) > 0).all() and ((top >= s) & (top < s + n_cand)).all()
    key = sc[:n_cand] if p.pool_kernel == 1 else oracle.pool(sc, n_cand, p.pool_kernel, p.pool_mode)
    brute = np.sort(np.lexsort((np.arange(n_cand), -key))[:n_take]) + s
    assert np.array_equal(top, brute)
    # outputs: a softmax average of the values each head attends to
    window = np.arange(L - min(w, L), L)
    sel = np.concatenate([top - s, window]).astype(np.int64)
    V = np.concatenate([p.sink_v, p.coeff_v[sel] @ p.basis_v.T])
    if V.shape[0]:
        for h in range(Hq):
            g = h // G
            Vg = V[:, g * dh:(g + 1) * dh]
            span = np.abs(Vg).max() + 1.0
            assert (out[h] >= Vg.min(axis=0) - 1e-12 * span).all() and (out[h] <= Vg.max(axis=0) + 1e-12 * span).all()
    # the twin: the same scores and, on the same selection, the same outputs
    sc_t = twin.scores(p)
    if L:
        assert np.abs(sc_t - sc).max() <= 1e-12 * max(1.0, np.abs(sc).max())
    assert np.array_equal(twin.select(p, sc), idx)
    ref = max(1.0, np.abs(out).max()) if out.size else 1.0
    assert np.abs(twin.decode_given_idx(p, idx) - out).max() <= 1e-12 * ref
