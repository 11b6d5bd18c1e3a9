"""NumPy twin of the fp64 decode oracle -- TEST INFRASTRUCTURE ONLY.

A second, independent reading of the same definitions as ``s4r_oracle.c``,
written with whole-array NumPy operations (matrix products, row-wise
reductions, a lexicographic sort) instead of the C file's loops.  It exists
to cross-check the C oracle (``tests/test_oracle_twin.py``: agreement to
1e-12 on small problems, identical selections); nothing else uses it, and the
product library never imports it.  It reuses only the ``Problem`` container
and the mode constants of ``oracle/__init__.py``, which hold no arithmetic.

Method source: the S4R review page ("S^4R: Selective Sampling, Subspaces, and
Sparse Reconstruction for Compressed Long-Context KV Caching", arXiv
2608.00528): Eq. 3 (encode), Eqs. 8-10 (latent scores), the free parameters
(pooling kernel 7), Eqs. 13-15 (selection with the local window kept),
Eqs. 16-18 (rebuilt rows and exact attention; sinks kept uncompressed).
The readings the page leaves open are those of the C oracle: CONCAT rows
(or per-head rows), scale 1/sqrt(r), softmax over all coefficient rows,
scores summed over rows, same-padded pooling over the candidates only
(average over the in-range neighbours), ties to the lower position.
"""
from __future__ import annotations

import numpy as np

from . import POOL_AVG, POOL_MAX, ROWS_CONCAT, ROWS_PER_HEAD, Problem

__all__ = ["encode", "reconstruct", "query_rows", "scores", "pool", "select", "decode_given_idx", "decode_step"]


def encode(states, basis) -> np.ndarray:
    """Coefficients C = S B (Eq. 3)."""
    return np.asarray(states, dtype=np.float64) @ np.asarray(basis, dtype=np.float64)


def reconstruct(coeffs, basis) -> np.ndarray:
    """Rebuilt rows C B^T (Eq. 16)."""
    return np.asarray(coeffs, dtype=np.float64) @ np.asarray(basis, dtype=np.float64).T


def query_rows(p: Problem) -> np.ndarray:
    """Rows of C_Q ("Core claim": queries projected into the key subspace).
    CONCAT: for each window slot w and in-group head j, the D'-vector of head
    j of every kv group, times B^K (W*G rows).  PER_HEAD: each head's query
    times the d_h rows of B^K of its kv group (W*H_q rows)."""
    W, Hq, dh = p.q.shape
    G = Hq // p.n_heads_kv
    if p.row_mode == ROWS_CONCAT:
        # q[w][g*G + j] -> q4[w][g][j]; row (w, j) is concat over g
        q4 = p.q.reshape(W, p.n_heads_kv, G, dh)
        rows = q4.transpose(0, 2, 1, 3).reshape(W * G, p.n_heads_kv * dh)
        return rows @ p.basis_k
    if p.row_mode == ROWS_PER_HEAD:
        g_of = np.arange(Hq) // G
        Bg = p.basis_k.reshape(p.n_heads_kv, dh, p.rank_k)[g_of]          # [H_q][d_h][r]
        return np.einsum("whd,hdr->whr", p.q, Bg).reshape(W * Hq, p.rank_k)
    raise ValueError("row_mode")


def scores(p: Problem) -> np.ndarray:
    """score_i = sum over the rows of the row's softmax probability of i,
    with logits C_Q . C_K[i] / sqrt(r_k) (Eqs. 8-10)."""
    if p.n_coeff == 0:
        return np.zeros(0)
    z = query_rows(p) @ p.coeff_k.T / np.sqrt(p.rank_k)                  # [R][L_c]
    e = np.exp(z - z.max(axis=1, keepdims=True))
    return (e / e.sum(axis=1, keepdims=True)).sum(axis=0)


def pool(score_vec, n_cand: int, kernel: int, mode: int = POOL_MAX) -> np.ndarray:
    """Stride-1, same-padded pooling of width `kernel` over the first
    n_cand scores; positions outside [0, n_cand) are left out (the average
    divides by the number of in-range neighbours)."""
    if kernel < 1 or kernel % 2 == 0 or mode not in (POOL_MAX, POOL_AVG):
        raise ValueError("pool")
    s = np.asarray(score_vec, dtype=np.float64)[:n_cand]
    if n_cand == 0:
        return np.zeros(0)
    half = kernel // 2
    pad = np.full(half, np.nan)
    win = np.lib.stride_tricks.sliding_window_view(np.concatenate([pad, s, pad]), kernel)   # [n_cand][kernel]
    return np.nanmax(win, axis=1) if mode == POOL_MAX else np.nanmean(win, axis=1)


def select(p: Problem, score_vec) -> np.ndarray:
    """Top-k absolute positions among the candidates i < L_c - w (larger
    score first, lower position on ties), ascending, -1 padded (Eqs. 13-15)."""
    n_cand = max(p.n_coeff - p.local_window, 0)
    key = np.asarray(score_vec, dtype=np.float64)[:n_cand]
    if p.pool_kernel > 1:
        key = pool(key, n_cand, p.pool_kernel, p.pool_mode)
    order = np.lexsort((np.arange(n_cand), -key))                        # score desc, then position asc
    take = np.sort(order[: min(p.top_k, n_cand)]) + p.n_sink
    out = np.full(p.top_k, -1, dtype=np.int32)
    out[: take.size] = take
    return out


def decode_given_idx(p: Problem, idx) -> np.ndarray:
    """Attention of the current query (window slot W - 1) of every head over
    the sinks and the rebuilt rows of the selection (the given top-k
    positions and the local window), Eqs. 16-18; out [H_q][d_h]."""
    W, Hq, dh = p.q.shape
    G = Hq // p.n_heads_kv
    L = p.n_coeff
    top = np.asarray(idx, dtype=np.int64)
    top = top[top >= 0] - p.n_sink
    window = np.arange(L - min(p.local_window, L), L)
    sel = np.concatenate([top, window]).astype(np.int64)
    K = np.concatenate([p.sink_k, reconstruct(p.coeff_k[sel], p.basis_k)])   # [s + n_sel][D']
    V = np.concatenate([p.sink_v, reconstruct(p.coeff_v[sel], p.basis_v)])
    out = np.zeros((Hq, dh))
    if K.shape[0] == 0:
        return out
    for h in range(Hq):
        g = h // G
        logits = K[:, g * dh:(g + 1) * dh] @ p.q[W - 1, h] / np.sqrt(dh)
        w = np.exp(logits - logits.max())
        out[h] = (w / w.sum()) @ V[:, g * dh:(g + 1) * dh]
    return out


def decode_step(p: Problem):
    """One decode step: (out [H_q][d_h], idx [top_k], scores [L_c])."""
    sc = scores(p)
    idx = select(p, sc)
    return decode_given_idx(p, idx), idx, sc
