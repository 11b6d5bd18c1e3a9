"""Test helpers: build decode problems from the seeded generator, run them
through the library's C ABI and through the oracle, and compare.

Coefficient caches are inputs of the decode path; the tests make them with a
float64 torch matmul on the CPU (states . basis, rounded to the storage type),
never with the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import oracle
import synth

# Comparators (one place, used by every parity test):
IDX_REL_TOL = 1e-6          # index swaps allowed only between scores this close (relative to tau)
OUT_TOL = {"bf16": (2e-2, 2e-3), "f32": (1e-4, 1e-4)}   # (max-abs, mean-abs)
SCORE_REL_TOL = {"bf16": 5e-6, "f32": 5e-6}             # GPU scores vs fp64 oracle (relative to max)


@dataclass
class Batch:
    dtype: str
    n_heads_kv: int
    local_window: int
    top_k: int
    pool_kernel: int
    row_mode: int
    pool_mode: int
    lengths: list            # L_c per problem
    cache_rows: int
    q: torch.Tensor          # [B][W][H_q][d_h] stored
    coeff_k: torch.Tensor    # [B][cache_rows][r_k] stored
    coeff_v: torch.Tensor
    basis_k: torch.Tensor    # [B][D'][r_k] stored
    basis_v: torch.Tensor
    sink_k: torch.Tensor     # [B][s][D'] stored
    sink_v: torch.Tensor

    @property
    def batch(self):
        return self.q.shape[0]

    def oracle_problem(self, b: int) -> oracle.Problem:
        L = self.lengths[b]
        f = lambda t: t.double().numpy()
        return oracle.Problem(q=f(self.q[b]), coeff_k=f(self.coeff_k[b, :L]), coeff_v=f(self.coeff_v[b, :L]),
                              basis_k=f(self.basis_k[b]), basis_v=f(self.basis_v[b]),
                              sink_k=f(self.sink_k[b]), sink_v=f(self.sink_v[b]),
                              n_heads_kv=self.n_heads_kv, local_window=self.local_window,
                              top_k=self.top_k, pool_kernel=self.pool_kernel, row_mode=self.row_mode,
                              pool_mode=self.pool_mode)


def encode_cpu(states: torch.Tensor, basis: torch.Tensor, dtype: str) -> torch.Tensor:
    """Input preparation: coefficients of stored states, fp64 matmul, then rounded."""
    return synth.store(states.double() @ basis.double(), dtype)


def make_batch(w: synth.Workload, *, lengths=None, layer=0, step=0, rank_k=None, rank_v=None,
               n_sink=None, local_window=None, top_k=None, query_window=None, pool_kernel=1,
               row_mode=0, cache_rows=None, tag="", pool_mode=0, windows=None):
    """Problems of workload `w` (shapes overridable), stored on the CPU.
    With windows = [t0, t1, ...] the query stream covers every listed decode
    step and the result is (batch at step t0, {t: q of step t})."""
    lengths = list(lengths if lengths is not None else synth.lengths(w))
    s = w.n_sink if n_sink is None else n_sink
    rk = rank_k or w.rank
    rv = rank_v or w.rank
    W = query_window or w.query_window
    qs, cks, cvs, bks, bvs, sks, svs, Lc = [], [], [], [], [], [], [], []
    steps = list(windows) if windows is not None else [step]
    q_by_step = {t: [] for t in steps}
    for b, L in enumerate(lengths):
        ww = synth.Workload(**{**w.__dict__, "n_sink": s})
        pin = synth.problem_inputs(ww, layer, b, L=L + s, n_query_rows=max(steps) + W, rank=max(rk, rv),
                                   tag=tag)
        for t in steps:
            q_by_step[t].append(pin.window(t, W))
        Bk, Bv = pin.basis_k[:, :rk].contiguous(), pin.basis_v[:, :rv].contiguous()
        cks.append(encode_cpu(pin.states_k[s:], Bk, w.dtype))
        cvs.append(encode_cpu(pin.states_v[s:], Bv, w.dtype))
        bks.append(Bk)
        bvs.append(Bv)
        sks.append(pin.states_k[:s])
        svs.append(pin.states_v[:s])
        qs.append(pin.window(steps[0], W))
        Lc.append(L)
    cap = cache_rows if cache_rows is not None else max(Lc + [1])
    B = len(lengths)
    sdt = synth.storage_dtype(w.dtype)
    ck = torch.zeros(B, cap, rk, dtype=sdt)
    cv = torch.zeros(B, cap, rv, dtype=sdt)
    for b in range(B):
        ck[b, :Lc[b]] = cks[b]
        cv[b, :Lc[b]] = cvs[b]
    batch = Batch(w.dtype, w.n_heads_kv, w.local_window if local_window is None else local_window,
                  w.top_k if top_k is None else top_k, pool_kernel, row_mode, pool_mode, Lc, cap,
                  torch.stack(qs), ck, cv, torch.stack(bks), torch.stack(bvs), torch.stack(sks),
                  torch.stack(svs))
    if windows is None:
        return batch
    return batch, {t: torch.stack(v) for t, v in q_by_step.items()}


def run_gpu(batch: Batch, device="cuda", want_scores=True, workspace=None):
    """Run one decode step of the batch through the C ABI; returns CPU tensors.
    A fresh, initialised workspace is used unless the caller passes one."""
    import rank_decode_attention_b200 as s4r
    dev = lambda t: t.to(device).contiguous()
    q, ck, cv, bk, bv, sk, sv = map(dev, (batch.q, batch.coeff_k, batch.coeff_v, batch.basis_k,
                                          batch.basis_v, batch.sink_k, batch.sink_v))
    B, W, Hq, dh = batch.q.shape
    lengths = torch.tensor(batch.lengths, dtype=torch.int32, device=device)
    out = torch.full((B, Hq, dh), float("nan"), dtype=torch.float32, device=device)
    idx = torch.full((B, max(batch.top_k, 1)), -7, dtype=torch.int32, device=device)
    scores = torch.full((B, batch.cache_rows), float("nan"), device=device) if want_scores else None
    kw = dict(q=q, coeff_k=ck, coeff_v=cv, basis_k=bk, basis_v=bv, sink_k=sk, sink_v=sv,
              lengths=lengths, n_heads_kv=batch.n_heads_kv, local_window=batch.local_window,
              top_k=batch.top_k, out=out, idx=idx, scores=scores, pool_kernel=batch.pool_kernel,
              pool_mode=batch.pool_mode, row_mode=batch.row_mode)
    nbytes = s4r.s4r_decode_workspace_bytes(s4r.decode_args(**kw))
    assert nbytes > 0
    ws = workspace
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        s4r.s4r_workspace_init(ws)
    assert ws.numel() >= nbytes
    s4r.s4r_decode_step(s4r.decode_args(**kw, workspace=ws))
    status = s4r.s4r_read_device_status(ws)
    torch.cuda.synchronize()
    return dict(out=out.cpu(), idx=idx[:, :batch.top_k].cpu(),
                scores=scores.cpu() if scores is not None else None, status=status)


def workspace_for(batch: Batch, device="cuda"):
    """A zeroed workspace large enough for one decode step of `batch`."""
    import rank_decode_attention_b200 as s4r
    B, W, Hq, dh = batch.q.shape
    a = s4r.DecodeArgs()
    a.batch, a.n_heads_q, a.n_heads_kv, a.head_dim = B, Hq, batch.n_heads_kv, dh
    a.rank_k, a.rank_v = batch.coeff_k.shape[2], batch.coeff_v.shape[2]
    a.n_sink, a.local_window, a.top_k, a.query_window = batch.sink_k.shape[1], batch.local_window, batch.top_k, W
    a.pool_kernel, a.pool_mode, a.row_mode = batch.pool_kernel, batch.pool_mode, batch.row_mode
    a.dtype = s4r.S4R_BF16 if batch.dtype == "bf16" else s4r.S4R_F32
    a.cache_rows = batch.cache_rows
    ws = torch.empty(s4r.s4r_decode_workspace_bytes(a), dtype=torch.uint8, device=device)
    s4r.s4r_workspace_init(ws)
    return ws


def ranking_scores(p: oracle.Problem, sc: np.ndarray) -> np.ndarray:
    """Scores the selection ranks by (pooled when pooling is on), candidates only."""
    n_cand = max(0, p.n_coeff - p.local_window)
    if p.pool_kernel > 1:
        return oracle.pool(sc, n_cand, p.pool_kernel, p.pool_mode)
    return sc[:n_cand]


def check_indices(gpu_idx: np.ndarray, ref_idx: np.ndarray, rank_sc: np.ndarray, n_sink: int,
                  tol=IDX_REL_TOL):
    """Index sets equal except for swaps between candidates whose fp64 scores
    are within `tol` of the k-th score tau."""
    g = gpu_idx[gpu_idx >= 0]
    r = ref_idx[ref_idx >= 0]
    assert np.all(np.diff(g) > 0), "GPU indices must be strictly ascending"
    assert g.size == r.size, f"selected count {g.size} != {r.size}"
    assert np.all(gpu_idx[g.size:] == -1), "padding must be -1"
    if g.size == 0:
        return 0
    assert g.min() >= n_sink and g.max() < n_sink + rank_sc.size, "index outside the candidates"
    tau = rank_sc[r - n_sink].min()
    only_g = np.setdiff1d(g, r)
    only_r = np.setdiff1d(r, g)
    assert np.all(rank_sc[only_g - n_sink] >= tau * (1 - tol)), \
        f"GPU-only indices {only_g[:8]} score below tau(1-tol)"
    assert np.all(rank_sc[only_r - n_sink] <= tau * (1 + tol)), \
        f"oracle-only indices {only_r[:8]} score above tau(1+tol)"
    return only_g.size


def check_batch(batch: Batch, res: dict, check_scores=True, score_rel_tol=None):
    """Compare one GPU decode step against the oracle, problem by problem.
    score_rel_tol overrides the score tolerance (cases with very wide logits,
    whose fp32 error grows with |logit|)."""
    max_abs, mean_abs = OUT_TOL[batch.dtype]
    stats = []
    for b in range(batch.batch):
        p = batch.oracle_problem(b)
        out_ref, idx_ref, sc_ref = oracle.decode_step(p)
        gi = res["idx"][b].numpy()
        swaps = check_indices(gi, idx_ref, ranking_scores(p, sc_ref), p.n_sink)
        if check_scores and res["scores"] is not None and p.n_coeff > 0:
            gs = res["scores"][b, :p.n_coeff].double().numpy()
            err = np.abs(gs - sc_ref).max() / max(sc_ref.max(), 1e-300)
            tol = SCORE_REL_TOL[batch.dtype] if score_rel_tol is None else score_rel_tol
            assert err < tol, f"problem {b}: score error {err:.3e} (tolerance {tol:.1e})"
        out_g = res["out"][b].double().numpy()
        out_at_gpu_idx = oracle.decode_given_idx(p, gi)
        d = np.abs(out_g - out_at_gpu_idx)
        assert np.isfinite(out_g).all(), "non-finite output"
        assert d.max() <= max_abs and d.mean() <= mean_abs, \
            f"problem {b}: out error max {d.max():.3e} mean {d.mean():.3e}"
        if swaps == 0:
            d2 = np.abs(out_g - out_ref)
            assert d2.max() <= max_abs and d2.mean() <= mean_abs
        stats.append((swaps, float(d.max())))
    return stats
