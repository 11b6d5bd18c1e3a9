"""Pins of the basis oracle (oracle/basis.py) to facts outside itself.

Hand-worked sample index sets and small SVDs (tests/golden/basis_examples.json),
closed forms of the normalised sample (its squared singular values add up to
its number of non-zero rows), exact recovery of a known low-rank row space,
the Eckart-Young optimality of the truncated SVD, and invariances the
definition implies.  CPU only.

S4R_BASIS_ORACLE may name another copy of the module (the mutant tests plant
mistakes in copies and expect this file to fail on them).
"""
import importlib.util
import json
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
_PATH = os.environ.get("S4R_BASIS_ORACLE") or os.path.join(ROOT, "oracle", "basis.py")
_spec = importlib.util.spec_from_file_location("oracle_basis_under_test", _PATH)
ob = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(ob)

GOLDEN = json.load(open(os.path.join(ROOT, "tests", "golden", "basis_examples.json")))


@pytest.mark.parametrize("case", GOLDEN["samples"], ids=lambda c: f"L{c['L']}-s{c['n_sink']}-T{c['n_sample']}")
def test_sample_rows_hand_worked(case):
    rows = ob.sample_rows(case["L"], case["n_sink"], case["n_sample"])
    assert rows.tolist() == case["rows"]


@pytest.mark.parametrize("seed", range(20))
def test_sample_rows_properties(seed):
    rng = np.random.default_rng(seed)
    s = int(rng.integers(0, 8))
    L = int(rng.integers(s, 5000))
    T = int(rng.integers(0, 700))
    rows = ob.sample_rows(L, s, T)
    n = min(T, L - s)
    assert len(rows) == n
    assert len(set(rows.tolist())) == n and np.all(np.diff(rows) > 0) if n > 1 else True
    if n:
        assert rows.min() >= s and rows.max() == L - 1
    n_recent = int(np.floor(0.7 * n + 0.5 + 1e-9))      # round half up of 0.7 n
    assert rows[n - n_recent:].tolist() == list(range(L - n_recent, L))
    uni = rows[:n - n_recent]
    if len(uni):
        assert uni[0] == s and uni[-1] < L - n_recent
        span = L - s - n_recent
        gaps = np.diff(np.append(uni, s + span))      # even spread: gaps differ by at most one
        assert gaps.max() - gaps.min() <= 1


@pytest.mark.parametrize("case", GOLDEN["svd"], ids=lambda c: f"{len(c['states'])}x{len(c['states'][0])}-r{c['rank']}")
def test_svd_hand_worked(case):
    B, sig, _ = ob.build_basis(np.array(case["states"]), case["L"], case["n_sink"], case["n_sample"], case["rank"])
    np.testing.assert_allclose(sig, case["sigma"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(B, np.array(case["basis"]), rtol=0, atol=1e-14)


def _states(L, D, seed, k=None):
    rng = np.random.default_rng(seed)
    if k is None:
        return rng.standard_normal((L, D)) * rng.uniform(0.1, 10, size=(L, 1))
    Q, _ = np.linalg.qr(rng.standard_normal((D, k)))
    return rng.standard_normal((L, k)) @ Q.T, Q


@pytest.mark.parametrize("L,D,T,zero", [(300, 64, 40, 0), (300, 32, 100, 3), (50, 96, 200, 5)])
def test_squared_singular_values_count_rows(L, D, T, zero):
    X = _states(L, D, 1)
    rows = ob.sample_rows(L, 4, T)
    X[rows[:zero]] = 0.0                                 # zero rows stay zero
    n = len(rows)
    _, sig, _ = ob.build_basis(X, L, 4, T, min(n, D))
    assert abs((sig ** 2).sum() - (n - zero)) < 1e-10 * n


@pytest.mark.parametrize("D,k", [(64, 8), (128, 32), (40, 40)])
def test_exact_low_rank_row_space_recovered(D, k):
    X, Q = _states(600, D, 2, k)
    B, sig, _ = ob.build_basis(X, 600, 4, 3 * k, k)
    assert np.abs(B @ B.T - Q @ Q.T).max() < 1e-10
    assert sig[-1] > 1e-6


@pytest.mark.parametrize("seed", range(4))
def test_truncation_is_eckart_young_optimal(seed):
    L, D, T, r = 400, 48, 60, 12
    X = _states(L, D, 10 + seed)
    B, sig, rows = ob.build_basis(X, L, 4, T, r)
    A = X[rows] / np.linalg.norm(X[rows], axis=1, keepdims=True)
    captured = np.linalg.norm(A @ B) ** 2
    assert abs(captured - (sig ** 2).sum()) < 1e-10 * captured
    rng = np.random.default_rng(seed)
    for _ in range(50):
        Y, _ = np.linalg.qr(rng.standard_normal((D, r)))
        assert np.linalg.norm(A @ Y) ** 2 <= captured + 1e-10
    # the next direction captures no more than the last kept one
    _, sig_all, _ = ob.build_basis(X, L, 4, T, min(len(rows), D))
    assert np.all(np.diff(sig_all) <= 0)


def test_orthonormal_ordered_and_signed():
    X = _states(500, 80, 3)
    B, sig, _ = ob.build_basis(X, 500, 4, 120, 40)
    assert np.abs(B.T @ B - np.eye(40)).max() < 1e-12
    assert np.all(np.diff(sig) <= 0)
    for k in range(40):
        d = int(np.argmax(np.abs(B[:, k])))
        assert B[d, k] > 0


def test_row_scale_sinks_and_unsampled_rows_do_not_matter():
    L, D, s, T, r = 400, 32, 4, 50, 10
    X = _states(L, D, 4)
    B, sig, rows = ob.build_basis(X, L, s, T, r)
    Y = X.copy()
    Y[rows] *= np.random.default_rng(5).uniform(0.01, 100, size=(len(rows), 1))   # token-wise scale
    Y[:s] = 1e6                                                                     # sink rows
    other = np.setdiff1d(np.arange(s, L), rows)
    Y[other] = -3.0                                                                 # rows not sampled
    B2, sig2, _ = ob.build_basis(Y, L, s, T, r)
    np.testing.assert_allclose(B2, B, atol=1e-10)
    np.testing.assert_allclose(sig2, sig, atol=1e-12)
    Y[rows[0]] = np.random.default_rng(6).standard_normal(D)                        # a sampled row does matter
    B3, _, _ = ob.build_basis(Y, L, s, T, r)
    assert np.abs(B3 @ B3.T - B @ B.T).max() > 1e-6


def test_rank_above_sample_or_width_is_refused():
    X = _states(30, 16, 7)
    with pytest.raises(ValueError):
        ob.build_basis(X, 30, 4, 10, 11)     # 10 sampled rows
    with pytest.raises(ValueError):
        ob.build_basis(X, 30, 4, 26, 17)     # D' = 16
