"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against a library routine, a closed form, an
invariant or a brute force that the definitions on the S4R review page
("S^4R: Selective Sampling, Subspaces, and Sparse Reconstruction for Compressed
Long-Context KV Caching", arXiv 2608.00528) fix:

  encode (Eq. 3)           -> BLAS matmul; exact recovery of in-span states
  rebuild (Eq. 16)         -> BLAS matmul; encode/rebuild round trip
  scoring (Eqs. 8-10)      -> torch SDPA weights (value = identity) when the
                              basis is a full rotation; conservation; rotation
                              invariance; single-row monotone reduction
  pooling                  -> torch max_pool1d / avg_pool1d (padding left out of
                              the count); a hand-worked average
  selection (Eqs. 13-15)   -> numpy stable lexsort brute force, forced ties
  attention (Eqs. 16-18)   -> torch SDPA (GQA) over all keys when nothing is
                              dropped; sinks-only case; convexity
  whole chain              -> two hand-worked examples (tests/golden)
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def rand_orthonormal(rng, rows, cols):
    q, r = np.linalg.qr(rng.standard_normal((rows, cols)))
    return q * np.sign(np.diag(r))[None, :]


def make_problem(rng, *, W=3, Hq=4, Hkv=2, dh=8, r=None, L=40, s=2, w=5, k=6, pool=1,
                 row_mode=oracle.ROWS_CONCAT, full_rank=False, pool_mode=oracle.POOL_MAX):
    Dp = Hkv * dh
    r = Dp if full_rank else (r or 6)
    K = rng.standard_normal((L, Dp))
    V = rng.standard_normal((L, Dp))
    if full_rank:
        Bk, Bv = rand_orthonormal(rng, Dp, Dp), rand_orthonormal(rng, Dp, Dp)
    else:
        Bk, Bv = rand_orthonormal(rng, Dp, r), rand_orthonormal(rng, Dp, r)
    p = oracle.Problem(q=rng.standard_normal((W, Hq, dh)), coeff_k=K @ Bk, coeff_v=V @ Bv,
                       basis_k=Bk, basis_v=Bv, sink_k=rng.standard_normal((s, Dp)),
                       sink_v=rng.standard_normal((s, Dp)), n_heads_kv=Hkv, local_window=w,
                       top_k=k, pool_kernel=pool, row_mode=row_mode, pool_mode=pool_mode)
    return p, K, V


# ---------------------------------------------------------------- encode / rebuild

def test_encode_matches_blas():
    rng = np.random.default_rng(1)
    S, B = rng.standard_normal((37, 24)), rng.standard_normal((24, 10))
    np.testing.assert_allclose(oracle.encode(S, B), S @ B, rtol=1e-13, atol=1e-13)


def test_encode_recovers_in_span_states():
    rng = np.random.default_rng(2)
    B = rand_orthonormal(rng, 32, 12)
    X = rng.standard_normal((50, 12))
    np.testing.assert_allclose(oracle.encode(X @ B.T, B), X, atol=1e-12)


def test_reconstruct_matches_blas_and_round_trips():
    rng = np.random.default_rng(3)
    C, B = rng.standard_normal((19, 7)), rng.standard_normal((21, 7))
    np.testing.assert_allclose(oracle.reconstruct(C, B), C @ B.T, rtol=1e-13, atol=1e-13)
    Bo = rand_orthonormal(rng, 21, 7)
    S = rng.standard_normal((19, 7)) @ Bo.T          # states inside span(Bo)
    np.testing.assert_allclose(oracle.reconstruct(oracle.encode(S, Bo), Bo), S, atol=1e-12)


# ---------------------------------------------------------------- scoring

def sdpa_weights(qrows, keys, scale):
    """Row-softmax weights from torch SDPA with an identity value matrix."""
    q = torch.from_numpy(qrows)[None, None]
    kk = torch.from_numpy(keys)[None, None]
    eye = torch.eye(keys.shape[0], dtype=torch.float64)[None, None]
    return F.scaled_dot_product_attention(q, kk, eye, scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("row_mode", [oracle.ROWS_CONCAT, oracle.ROWS_PER_HEAD])
def test_scores_full_rotation_equal_sdpa_weights(row_mode):
    """With B a full rotation (r = D') the latent logits equal the exact ones."""
    rng = np.random.default_rng(4)
    W, Hq, Hkv, dh = 3, 6, 2, 4
    G, Dp = Hq // Hkv, Hkv * dh
    p, K, _ = make_problem(rng, W=W, Hq=Hq, Hkv=Hkv, dh=dh, L=33, full_rank=True, row_mode=row_mode)
    got = oracle.scores(p)
    if row_mode == oracle.ROWS_CONCAT:
        # row (w, j): concatenation over groups g of head g*G + j
        rows = np.stack([np.concatenate([p.q[w, g * G + j] for g in range(Hkv)])
                         for w in range(W) for j in range(G)])
        want = sdpa_weights(rows, K, 1.0 / math.sqrt(Dp)).sum(0)
    else:
        want = np.zeros(K.shape[0])
        for w in range(W):
            for h in range(Hq):
                g = h // G
                want += sdpa_weights(p.q[w, h][None], K[:, g * dh:(g + 1) * dh],
                                     1.0 / math.sqrt(Dp))[0]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("row_mode,n_rows", [(oracle.ROWS_CONCAT, 3 * 2), (oracle.ROWS_PER_HEAD, 3 * 4)])
def test_scores_conserve_row_mass(row_mode, n_rows):
    rng = np.random.default_rng(5)
    p, _, _ = make_problem(rng, W=3, Hq=4, Hkv=2, L=57, row_mode=row_mode)
    assert abs(oracle.scores(p).sum() - n_rows) < 1e-12


def test_scores_single_row_reduce_to_exact_attention_weights():
    """W = G = H_kv = 1, low rank: score = softmax(q . k_hat / sqrt(r))."""
    rng = np.random.default_rng(6)
    p, _, _ = make_problem(rng, W=1, Hq=1, Hkv=1, dh=16, r=5, L=45)
    khat = p.coeff_k @ p.basis_k.T
    want = sdpa_weights(p.q[0], khat, 1.0 / math.sqrt(p.rank_k))[0]
    np.testing.assert_allclose(oracle.scores(p), want, rtol=1e-12, atol=1e-15)


def test_rotation_invariance_of_the_latent_space():
    rng = np.random.default_rng(7)
    p, _, _ = make_problem(rng, L=60, r=6, k=8, w=4)
    out0, idx0, sc0 = oracle.decode_step(p)
    R = rand_orthonormal(rng, 6, 6)
    p2 = oracle.Problem(q=p.q, coeff_k=p.coeff_k @ R, coeff_v=p.coeff_v @ R,
                        basis_k=p.basis_k @ R, basis_v=p.basis_v @ R, sink_k=p.sink_k,
                        sink_v=p.sink_v, n_heads_kv=p.n_heads_kv, local_window=4, top_k=8)
    out1, idx1, sc1 = oracle.decode_step(p2)
    np.testing.assert_allclose(sc1, sc0, rtol=1e-10)
    np.testing.assert_array_equal(idx1, idx0)
    np.testing.assert_allclose(out1, out0, atol=1e-10)


# ---------------------------------------------------------------- pooling + selection

@pytest.mark.parametrize("kernel", [3, 7])
def test_pool_matches_torch_max_pool(kernel):
    rng = np.random.default_rng(8)
    s = rng.random(41)
    want = F.max_pool1d(torch.from_numpy(s)[None, None], kernel, stride=1,
                        padding=kernel // 2)[0, 0].numpy()
    np.testing.assert_array_equal(oracle.pool(s, s.size, kernel), want)


@pytest.mark.parametrize("kernel", [3, 7])
def test_avg_pool_matches_torch_avg_pool_without_padding_in_the_count(kernel):
    rng = np.random.default_rng(18)
    s = rng.random(41)
    want = F.avg_pool1d(torch.from_numpy(s)[None, None], kernel, stride=1, padding=kernel // 2,
                        count_include_pad=False)[0, 0].numpy()
    np.testing.assert_allclose(oracle.pool(s, s.size, kernel, oracle.POOL_AVG), want, rtol=1e-15, atol=0)


def test_avg_pool_hand_worked():
    # kappa = 3 over [1, 2, 3, 4, 5]: the ends average two in-range neighbours,
    # (1 + 2) / 2 and (4 + 5) / 2; the middle ones three.
    got = oracle.pool(np.array([1.0, 2.0, 3.0, 4.0, 5.0]), 5, 3, oracle.POOL_AVG)
    np.testing.assert_array_equal(got, [1.5, 2.0, 3.0, 4.0, 4.5])
    # kappa = 7 over three candidates: every window covers all of them.
    got = oracle.pool(np.array([3.0, 0.0, 6.0]), 3, 7, oracle.POOL_AVG)
    np.testing.assert_array_equal(got, [3.0, 3.0, 3.0])


def brute_topk(scores, n_cand, k, s):
    # stable lexsort: primary key -score, secondary key position
    order = np.lexsort((np.arange(n_cand), -scores[:n_cand]))
    take = np.sort(order[:min(k, n_cand)]) + s
    return np.concatenate([take, -np.ones(k - take.size, dtype=np.int64)])


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    L, w, k, s = 50, 7, 9, 3
    p, _, _ = make_problem(rng, L=L, w=w, k=k, s=s)
    scores = np.round(rng.random(L) * 4) / 4          # heavy exact ties
    np.testing.assert_array_equal(oracle.select(p, scores), brute_topk(scores, L - w, k, s))


def test_select_with_pooling_uses_pooled_ranking():
    rng = np.random.default_rng(9)
    L, w, k, s = 64, 8, 10, 4
    p, _, _ = make_problem(rng, L=L, w=w, k=k, s=s, pool=5)
    scores = rng.random(L)
    pooled = F.max_pool1d(torch.from_numpy(scores[:L - w])[None, None], 5, 1, 2)[0, 0].numpy()
    want = brute_topk(np.concatenate([pooled, scores[L - w:]]), L - w, k, s)
    np.testing.assert_array_equal(oracle.select(p, scores), want)


def test_select_with_avg_pooling_uses_pooled_ranking():
    rng = np.random.default_rng(19)
    L, w, k, s = 64, 8, 10, 4
    p, _, _ = make_problem(rng, L=L, w=w, k=k, s=s, pool=7, pool_mode=oracle.POOL_AVG)
    scores = rng.random(L)
    pooled = F.avg_pool1d(torch.from_numpy(scores[:L - w])[None, None], 7, 1, 3,
                          count_include_pad=False)[0, 0].numpy()
    want = brute_topk(np.concatenate([pooled, scores[L - w:]]), L - w, k, s)
    np.testing.assert_array_equal(oracle.select(p, scores), want)


@pytest.mark.parametrize("L,w,k,expect_n", [(5, 8, 4, 0), (8, 8, 4, 0), (10, 8, 4, 2), (30, 8, 0, 0)])
def test_select_edge_cases(L, w, k, expect_n):
    rng = np.random.default_rng(10)
    p, _, _ = make_problem(rng, L=L, w=w, k=k, s=2)
    idx = oracle.select(p, rng.random(L))
    assert idx.shape == (k,)
    assert (idx >= 0).sum() == expect_n
    assert np.all(idx[expect_n:] == -1)
    if expect_n:
        assert np.all(np.diff(idx[:expect_n]) > 0) and idx[0] >= 2 and idx[expect_n - 1] < 2 + L - w


# ---------------------------------------------------------------- attention

def sdpa_gqa(qcur, keys, vals, Hkv):
    q = torch.from_numpy(qcur)[None, :, None, :]            # [1, Hq, 1, dh]
    dh = qcur.shape[-1]
    kk = torch.from_numpy(keys.reshape(-1, Hkv, dh).transpose(1, 0, 2).copy())[None]
    vv = torch.from_numpy(vals.reshape(-1, Hkv, dh).transpose(1, 0, 2).copy())[None]
    return F.scaled_dot_product_attention(q, kk, vv, enable_gqa=True)[0, :, 0, :].numpy()


def test_attention_reduces_to_full_attention():
    """r = D' and k + w >= L_c: the step is textbook attention over all L keys."""
    rng = np.random.default_rng(11)
    p, K, V = make_problem(rng, W=2, Hq=8, Hkv=2, dh=8, L=30, s=3, w=10, k=25, full_rank=True)
    out, idx, _ = oracle.decode_step(p)
    keys = np.concatenate([p.sink_k, K])
    vals = np.concatenate([p.sink_v, V])
    np.testing.assert_allclose(out, sdpa_gqa(p.q[-1], keys, vals, 2), atol=1e-10)
    assert sorted(idx[idx >= 0].tolist()) == list(range(3, 3 + 20))


def test_sinks_only_attention():
    rng = np.random.default_rng(12)
    p, _, _ = make_problem(rng, Hq=6, Hkv=3, dh=4, L=20, s=4, w=0, k=0)
    out = oracle.decode_given_idx(p, np.zeros(0, dtype=np.int32))
    np.testing.assert_allclose(out, sdpa_gqa(p.q[-1], p.sink_k, p.sink_v, 3), atol=1e-12)


def test_attention_output_is_convex_combination():
    rng = np.random.default_rng(13)
    p, _, _ = make_problem(rng, Hq=4, Hkv=2, dh=8, L=50, s=2, w=6, k=7)
    out, idx, _ = oracle.decode_step(p)
    rows = sorted(set((idx[idx >= 0] - 2).tolist()) | set(range(50 - 6, 50)))
    vhat = p.coeff_v[rows] @ p.basis_v.T
    allv = np.concatenate([p.sink_v, vhat])
    for h in range(4):
        g = h // 2
        sl = allv[:, g * 8:(g + 1) * 8]
        assert np.all(out[h] <= sl.max(0) + 1e-12) and np.all(out[h] >= sl.min(0) - 1e-12)


def test_needle_aligned_with_query_is_selected():
    rng = np.random.default_rng(14)
    p, _, _ = make_problem(rng, W=1, Hq=2, Hkv=1, dh=8, r=8, L=200, s=2, w=4, k=1)
    # plant a coefficient row parallel to the projected query, 3x larger than any other
    cq = sum(p.q[0, j] @ p.basis_k for j in range(2))
    ck = p.coeff_k.copy()
    ck[77] = 3 * np.abs(ck).max() * cq / np.linalg.norm(cq)
    p2 = oracle.Problem(q=p.q, coeff_k=ck, coeff_v=p.coeff_v, basis_k=p.basis_k, basis_v=p.basis_v,
                        sink_k=p.sink_k, sink_v=p.sink_v, n_heads_kv=1, local_window=4, top_k=1)
    _, idx, _ = oracle.decode_step(p2)
    assert idx.tolist() == [77 + 2]


# ---------------------------------------------------------------- hand-worked examples

def _closed(v):
    if isinstance(v, str):
        return float(eval(v, {"__builtins__": {}},
                          {"sqrt2": math.sqrt(2.0), "ln2": math.log(2.0), "ln3": math.log(3.0)}))
    return float(v)


def _arr(x):
    return np.vectorize(_closed, otypes=[np.float64])(np.array(x, dtype=object))


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    p = oracle.Problem(q=_arr(case["q"]), coeff_k=_arr(case["coeff_k"]), coeff_v=_arr(case["coeff_v"]),
                       basis_k=_arr(case["basis_k"]), basis_v=_arr(case["basis_v"]),
                       sink_k=_arr(case["sink_k"]), sink_v=_arr(case["sink_v"]),
                       n_heads_kv=case["n_heads_kv"], local_window=case["local_window"],
                       top_k=case["top_k"])
    out, idx, sc = oracle.decode_step(p)
    np.testing.assert_allclose(sc, _arr(case["scores"]), rtol=1e-14, atol=1e-15)
    assert idx.tolist() == case["idx"]
    np.testing.assert_allclose(out, _arr(case["out"]), rtol=1e-14, atol=1e-15)
