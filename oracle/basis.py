"""fp64 oracle of the S4R prefill bases -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the product library never calls it and
shares no code with it.

Source: "S^4R: Selective Sampling, Subspaces, and Sparse Reconstruction for
Compressed Long-Context KV Caching" (arXiv 2608.00528), review page:
"What carries the argument" and the Referee Report's summary (Eqs. 1-2: a
truncated SVD of a sampled, token-wise normalised set of non-sink states; the
top-r right singular vectors are the basis), "Core claim" (sink tokens are
kept apart; T' non-sink tokens are sampled with a 7:3 split between recent and
uniformly spaced positions) and the free-parameter list (the 7:3 split).

Readings where the page is silent (the same readings the CUDA path follows):
  * the sample has n = min(T', L - s) rows; the recent share is the last
    round(0.7 n) non-sink rows, rounded half up in exact integer arithmetic
    ((7 n + 5) div 10); the other n_u rows are spread evenly over the older
    non-sink rows [s, L - n_recent): row s + floor(j * span / n_u), j < n_u;
  * "token-wise normalised" scales each sampled row to unit Euclidean norm
    (an all-zero row stays zero);
  * the basis columns are ordered by decreasing singular value, and each is
    signed so that its entry of largest magnitude (lowest index on ties) is
    positive.  Only the spanned subspace matters to the decode path, but a
    fixed sign makes the output well defined.
The SVD itself is a library routine (numpy.linalg.svd), used as one step.
"""
from __future__ import annotations

import numpy as np


def sample_rows(L: int, n_sink: int, n_sample: int) -> np.ndarray:
    """Row indices of the 7:3 recent-to-uniform sample, ascending ("Core claim")."""
    if L < 0 or n_sink < 0 or n_sample < 0:
        raise ValueError("negative size")
    n_avail = max(0, L - n_sink)
    n = min(n_sample, n_avail)
    n_recent = (7 * n + 5) // 10
    n_uniform = n - n_recent
    span = n_avail - n_recent
    uniform = [n_sink + (j * span) // n_uniform for j in range(n_uniform)]
    recent = list(range(L - n_recent, L))
    return np.array(uniform + recent, dtype=np.int64)


def normalise_rows(A: np.ndarray) -> np.ndarray:
    """Each row scaled to unit Euclidean norm; zero rows stay zero."""
    A = np.asarray(A, dtype=np.float64)
    norms = np.sqrt((A * A).sum(axis=1))
    out = A.copy()
    nz = norms > 0
    out[nz] = A[nz] / norms[nz, None]
    return out


def sign_convention(B: np.ndarray) -> np.ndarray:
    """Flip each column so that its largest-magnitude entry (first on ties) is positive."""
    B = B.copy()
    for k in range(B.shape[1]):
        d = int(np.argmax(np.abs(B[:, k])))
        if B[d, k] < 0:
            B[:, k] = -B[:, k]
    return B


def build_basis(states: np.ndarray, L: int, n_sink: int, n_sample: int, rank: int):
    """Top-`rank` right singular vectors of the normalised sample (Eqs. 1-2).

    states: [>= L][D'] token states of one (sequence, layer, K or V) problem.
    Returns (B [D'][rank], sigma [rank], rows).  Raises ValueError when the
    sample has fewer than `rank` rows or `rank` exceeds D'.
    """
    states = np.asarray(states, dtype=np.float64)
    rows = sample_rows(L, n_sink, n_sample)
    d_model = states.shape[1]
    if rank > min(len(rows), d_model):
        raise ValueError(f"rank {rank} exceeds the sample's {len(rows)} rows or D' = {d_model}")
    A = normalise_rows(states[rows])
    _, s, vt = np.linalg.svd(A, full_matrices=False)
    B = sign_convention(vt[:rank].T)
    return np.ascontiguousarray(B), s[:rank].copy(), rows
