"""Seeded synthetic inputs for S4R decode (shared by the tests, smoke check and
benchmark).

This module draws inputs only.  It holds none of the decode or encode
arithmetic: coefficient caches are made by whoever consumes these inputs (the
oracle's encode on the CPU side, the library's own encode kernel on the GPU
side).  It never imports the oracle or the product library.

Recipe (one (sequence, layer) problem, float64 throughout):
  * states X = G . diag(sigma) . U^T + noise, G ~ N(0,1) of size L x t,
    sigma_i = i^-0.8 (i = 1..t), U an orthonormal D' x t matrix (QR of a
    Gaussian), noise ~ N(0, 0.05^2);
  * the first n_sink rows are scaled 10x (attention sinks);
  * needle rows are scaled 3x (8 uniform non-sink rows, or 64 rows in the
    middle 80% of positions for the long-context workload);
  * bases: 7:3 recent-to-uniform sample of non-sink rows, each row scaled to
    unit norm, top-r right singular vectors of the sample from a library SVD.
    This is the prefill step of the method, done here in float64 only to make
    realistic bases; bases are inputs of the decode path.
  * queries ~ N(0,1): a stream of rows [H_q][d_h]; decode step t uses stream
    rows t .. t+W-1 as its query window.

Generation runs in torch on the device it is given; the CPU and CUDA random
streams differ, so a problem is only reproducible on the same device kind.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import torch

F32 = "f32"
BF16 = "bf16"


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str
    batch: int              # independent sequences
    layers: int
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    prompt_len: int         # L (ignored when lengths are ragged)
    rank: int
    n_sink: int
    local_window: int
    top_k: int
    query_window: int
    steps: int
    true_rank: int
    n_sample: int
    n_needles: int
    needle_middle: bool = False
    ragged: tuple = ()      # (lo, hi) for U[lo, hi] lengths; empty = fixed
    append: bool = False    # each step first appends one encoded token
    pool_kernel: int = 1
    row_mode: int = 0       # scoring rows: 0 CONCAT (W * G), 1 per head (W * H_q)

    @property
    def d_model(self) -> int:
        return self.n_heads_kv * self.head_dim


WORKLOADS = {
    0: Workload("tiny-f32", F32, 1, 1, 4, 2, 64, 2048, 32, 4, 64, 128, 8, 1, 32, 256, 8),
    1: Workload("llama3-8b-shape-L32k", BF16, 1, 32, 32, 8, 128, 32768, 192, 4, 128, 1024, 16, 64,
                256, 256, 8),
    2: Workload("batched-16x8k", BF16, 16, 32, 32, 8, 128, 8192, 128, 4, 128, 512, 16, 128,
                256, 512, 8),
    3: Workload("long-context-128k", BF16, 1, 32, 32, 8, 128, 131072, 256, 4, 256, 2048, 16, 16,
                256, 256, 64, needle_middle=True),
    4: Workload("ragged-encode-decode", BF16, 8, 1, 32, 8, 128, 65536, 256, 4, 128, 1024, 16, 256,
                256, 256, 8, ragged=(4096, 65536), append=True),
}

BULK_ENCODE_TOKENS = 65536


def seed_of(*parts) -> int:
    """Stable 63-bit seed from a tuple of labels (workload, layer, sequence, tensor)."""
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def lengths(w: Workload, seed_label="lengths") -> list:
    """Prompt length L of each sequence (ragged draw when the workload asks)."""
    if not w.ragged:
        return [w.prompt_len] * w.batch
    g = generator(seed_of(w.name, seed_label), "cpu")
    lo, hi = w.ragged
    return [int(v) for v in torch.randint(lo, hi + 1, (w.batch,), generator=g)]


def orthonormal(rows: int, cols: int, gen: torch.Generator, device) -> torch.Tensor:
    a = torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float64)
    qm, rm = torch.linalg.qr(a)
    return qm * torch.sign(torch.diagonal(rm)).unsqueeze(0)


def states(L: int, d_model: int, true_rank: int, n_sink: int, n_needles: int,
           needle_middle: bool, seed: int, device="cpu") -> torch.Tensor:
    """Synthetic key or value states [L][D'] (float64), recipe in the module doc."""
    gen = generator(seed, device)
    t = min(true_rank, d_model)
    U = orthonormal(d_model, t, gen, device)
    sigma = torch.arange(1, t + 1, device=device, dtype=torch.float64).pow(-0.8)
    G = torch.randn(L, t, generator=gen, device=device, dtype=torch.float64)
    X = (G * sigma) @ U.T
    X += 0.05 * torch.randn(L, d_model, generator=gen, device=device, dtype=torch.float64)
    X[:n_sink] *= 10.0
    if n_needles and L > n_sink:
        if needle_middle:
            lo, hi = max(n_sink, int(0.1 * L)), max(n_sink + 1, int(0.9 * L))
        else:
            lo, hi = n_sink, L
        pos = lo + torch.randperm(hi - lo, generator=gen, device=device)[: min(n_needles, hi - lo)]
        X[pos] *= 3.0
    return X


def sample_rows(L: int, n_sink: int, n_sample: int) -> torch.Tensor:
    """7:3 recent-to-uniform sample of non-sink row indices (at most L - n_sink)."""
    n_avail = L - n_sink
    n_sample = min(n_sample, n_avail)
    n_recent = int(round(0.7 * n_sample))
    n_uniform = n_sample - n_recent
    recent = torch.arange(L - n_recent, L, dtype=torch.int64)
    span = n_avail - n_recent
    if n_uniform > 0 and span > 0:
        uniform = n_sink + (torch.arange(n_uniform, dtype=torch.int64) * span) // n_uniform
    else:
        uniform = torch.empty(0, dtype=torch.int64)
    return torch.cat([uniform, recent])


def basis(X: torch.Tensor, rows: torch.Tensor, rank: int, gen: torch.Generator | None = None) -> torch.Tensor:
    """Top-`rank` right singular vectors [D'][rank] of the unit-normalised sample.
    A sample with fewer rows than `rank` (a very short prompt) is completed
    with random orthonormal directions orthogonal to its span."""
    A = X[rows.to(X.device)]
    A = A / A.norm(dim=1, keepdim=True).clamp_min(1e-300)
    _, _, Vh = torch.linalg.svd(A, full_matrices=False)
    V = Vh[:rank].T
    if V.shape[1] < rank:
        extra = torch.randn(V.shape[0], rank - V.shape[1], generator=gen, device=X.device,
                            dtype=torch.float64)
        extra -= V @ (V.T @ extra)
        qm, rm = torch.linalg.qr(extra)
        V = torch.cat([V, qm * torch.sign(torch.diagonal(rm)).unsqueeze(0)], dim=1)
    return V.contiguous()


def queries(n_rows: int, n_heads_q: int, head_dim: int, seed: int, device="cpu") -> torch.Tensor:
    gen = generator(seed, device)
    return torch.randn(n_rows, n_heads_q, head_dim, generator=gen, device=device, dtype=torch.float64)


def storage_dtype(dtype: str) -> torch.dtype:
    return {F32: torch.float32, BF16: torch.bfloat16}[dtype]


def store(x: torch.Tensor, dtype: str) -> torch.Tensor:
    """Round float64 values to the storage type (via float32, round-to-nearest-even)."""
    return x.to(torch.float32).to(storage_dtype(dtype)).contiguous()


@dataclass
class ProblemInputs:
    """Stored (storage-dtype) inputs of one (sequence, layer) problem, before encode."""
    states_k: torch.Tensor    # [L][D'] stored; rows 0..s-1 are the sinks
    states_v: torch.Tensor
    basis_k: torch.Tensor     # [D'][r] stored
    basis_v: torch.Tensor
    q_stream: torch.Tensor    # [steps + W - 1][H_q][d_h] stored
    extras: dict = field(default_factory=dict)

    def window(self, step: int, W: int) -> torch.Tensor:
        return self.q_stream[step: step + W]


def problem_inputs(w: Workload, layer: int, seq: int, device="cpu", L: int | None = None,
                   n_query_rows: int | None = None, rank: int | None = None,
                   tag: str = "") -> ProblemInputs:
    """Draw one problem's stored inputs following the workload recipe."""
    L = L if L is not None else lengths(w)[seq]
    r = rank if rank is not None else w.rank
    base = (w.name + tag, layer, seq)
    Xk = states(L, w.d_model, w.true_rank, w.n_sink, w.n_needles, w.needle_middle,
                seed_of(*base, "k"), device)
    Xv = states(L, w.d_model, w.true_rank, w.n_sink, w.n_needles, w.needle_middle,
                seed_of(*base, "v"), device)
    rows = sample_rows(L, w.n_sink, w.n_sample)
    Bk = basis(Xk, rows, r, generator(seed_of(*base, "k-fill"), device))
    Bv = basis(Xv, rows, r, generator(seed_of(*base, "v-fill"), device))
    nq = n_query_rows if n_query_rows is not None else w.steps + w.query_window - 1
    Q = queries(nq, w.n_heads_q, w.head_dim, seed_of(*base, "q"), device)
    return ProblemInputs(store(Xk, w.dtype), store(Xv, w.dtype), store(Bk, w.dtype),
                         store(Bv, w.dtype), store(Q, w.dtype))
