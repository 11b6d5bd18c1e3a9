"""GPU parity of the decode step on the branches that ordinary inputs never
reach, through the C ABI against the fp64 oracle:

  * wide logit range: the tensor-core scoring kernel works in base 2 with
    e = 2^y; a 128-position tile in which some |y| exceeds 100 switches to
    per-row integer offsets 2^(y - k) so that nothing overflows or flushes.
    Each case first checks, from the stored inputs, that it really drives
    tiles past that limit (Eqs. 8-10, major comment 2, §3.2.2);
  * a bounded device wait that runs out: the scoring kernel's grid barrier
    (or per-problem arrival counter) is made unreachable through the
    library's test hook, the kernel gives up after a short limit and reports
    S4R_ERR_TIMEOUT, and the next call on the same workspace matches the
    oracle again;
  * average pooling of the candidate scores ("free parameters": kernel 7),
    with exact ties that pooling creates;
  * a cache with more candidates than the 8-CTA cluster select holds, which
    the single-CTA select takes (Eqs. 13-15).

Comparators are those of every decode parity test (tests/problems.py).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from problems import check_batch, make_batch, run_gpu, workspace_for

pytestmark = pytest.mark.gpu

W1 = synth.WORKLOADS[1]
RANGE_LIMIT = 100.0      # |y| beyond which a tile takes per-row offsets
TILE = 128


def concat_rows(batch, b):
    """C_Q of problem b from the stored inputs (CONCAT rows), fp64 [R][r]."""
    q = batch.q[b].double().numpy()                       # [W][H_q][d_h]
    W, Hq, dh = q.shape
    Hkv = batch.n_heads_kv
    G = Hq // Hkv
    qc = np.concatenate([q[:, g * G:(g + 1) * G, :] for g in range(Hkv)], axis=2)   # [W][G][D']
    return qc.reshape(W * G, Hkv * dh) @ batch.basis_k[b].double().numpy()


def per_head_rows(batch, b):
    """C_Q of problem b (PER_HEAD rows, row w * H_q + h): q[w][h] . B^K[g d_h ..
    (g + 1) d_h], g = h / G; fp64 [W H_q][r]."""
    q = batch.q[b].double().numpy()                       # [W][H_q][d_h]
    W, Hq, dh = q.shape
    G = Hq // batch.n_heads_kv
    bk = batch.basis_k[b].double().numpy()
    return np.stack([q[w, h] @ bk[(h // G) * dh:(h // G + 1) * dh] for w in range(W) for h in range(Hq)])


def base2_logits(batch, b):
    """y[row][i] = (C_Q[row] . C_K[i]) / sqrt(r) * log2(e), to check which
    branch a case reaches."""
    L = batch.lengths[b]
    ck = batch.coeff_k[b, :L].double().numpy()
    cq = per_head_rows(batch, b) if batch.row_mode == 1 else concat_rows(batch, b)
    return (cq @ ck.T) / np.sqrt(ck.shape[1]) * np.log2(np.e)


def tile_ranges(y):
    n_t = (y.shape[1] + TILE - 1) // TILE
    return np.array([np.abs(y[:, t * TILE:(t + 1) * TILE]).max() for t in range(n_t)])


def score_tol(y_max):
    """Score tolerance (relative to the largest score) for logits up to
    |y| = y_max.  The kernel forms each base-2 logit in fp32 from exact
    products, so its error is a few units of 2^-24 |y|; e = 2^(y - k) then
    carries ln(2) times that as relative error, and the row normalisers the
    same.  16 * 2^-24 * y_max covers both with margin; the usual 5e-6 stays
    the floor."""
    return 5e-6 + 16.0 * 2.0 ** -24 * y_max


def _run(batch, y_max=None):
    res = run_gpu(batch)
    assert res["status"] == 0, f"device status {res['status']}"
    return check_batch(batch, res, score_rel_tol=None if y_max is None else score_tol(y_max))


def test_wide_range_every_tile():
    # The query window scaled by a power of two (exact in bf16), the smallest
    # that takes every tile's largest |y| past 110: every tile is past the
    # limit, and some row's normaliser lies far above the fp32 range (2^k
    # with k over 128 before the offsets).
    batch = make_batch(W1, lengths=[5003], top_k=16, local_window=32, tag="wide-all")
    y0 = tile_ranges(base2_logits(batch, 0)).min()
    scale = 2.0 ** np.ceil(np.log2(110.0 / y0))
    batch = dataclasses.replace(batch, q=(batch.q.double() * scale).to(batch.q.dtype))
    y = base2_logits(batch, 0)
    ranges = tile_ranges(y)
    assert ranges.min() > RANGE_LIMIT, ranges.min()
    assert y.max(axis=1).max() > 128.0
    _run(batch, ranges.max())


def test_wide_range_every_tile_per_head_rows():
    # The per-head reading (W * H_q = 512 rows) takes the many-rows scoring
    # kernel (chunks of 64 rows, two passes); the same scaling drives every
    # tile past the limit, so both passes take the per-row offsets.
    batch = make_batch(W1, lengths=[3001], top_k=16, local_window=32, row_mode=1, tag="wide-heads")
    y0 = tile_ranges(base2_logits(batch, 0)).min()
    scale = 2.0 ** np.ceil(np.log2(110.0 / y0))
    batch = dataclasses.replace(batch, q=(batch.q.double() * scale).to(batch.q.dtype))
    ranges = tile_ranges(base2_logits(batch, 0))
    assert ranges.min() > RANGE_LIMIT, ranges.min()
    _run(batch, ranges.max())


def test_wide_range_some_tiles():
    # Two tiles' key coefficients (rows 1024 .. 1279) scaled by a power of two
    # so that their largest |y| is near 130 while every other tile stays
    # below the limit: wide and ordinary tiles meet in one problem, and the
    # scaled rows dominate every row's softmax.
    batch = make_batch(W1, lengths=[5003, 2100], top_k=32, local_window=64, tag="wide-some")
    y0 = tile_ranges(base2_logits(batch, 0))
    scale = 2.0 ** np.ceil(np.log2(130.0 / y0[8:10].max()))
    ck = batch.coeff_k.clone()
    ck[0, 1024:1280] = (ck[0, 1024:1280].double() * scale).to(ck.dtype)
    batch = dataclasses.replace(batch, coeff_k=ck)
    ranges = tile_ranges(base2_logits(batch, 0))
    assert ranges[8:10].max() > RANGE_LIMIT
    assert np.delete(ranges, [8, 9]).max() < RANGE_LIMIT
    assert tile_ranges(base2_logits(batch, 1)).max() < RANGE_LIMIT
    _run(batch, ranges.max())


def test_wide_range_rows_far_below_zero():
    # Every key row shifted by one vector along -d, d the unit mean direction
    # of the scoring rows: before rounding to bf16, each row's logits all move
    # by the same amount, down for the rows that point along d.  Rows whose
    # every logit lies below -126 have normalisers below the fp32 range.
    L = 3000
    batch = make_batch(W1, lengths=[L], top_k=16, local_window=16, tag="wide-neg")
    cq = concat_rows(batch, 0)
    d = cq.mean(axis=0)
    d /= np.linalg.norm(d)
    proj = cq @ d
    y0 = base2_logits(batch, 0)
    r = cq.shape[1]
    c = (250.0 + np.abs(y0).max()) * np.sqrt(r) / (proj.max() * np.log2(np.e))
    ck = batch.coeff_k[0, :L].double() - c * torch.from_numpy(d)[None, :]
    batch.coeff_k[0, :L] = synth.store(ck, "bf16")
    y = base2_logits(batch, 0)
    assert tile_ranges(y).min() > RANGE_LIMIT
    assert (y.max(axis=1) < -126.0).any()
    _run(batch, np.abs(y).max())


@pytest.mark.parametrize("lengths", [[5003], [5003, 777, 130]], ids=["one-problem", "three-problems"])
def test_bounded_wait_runs_out_and_the_next_call_recovers(lengths):
    # One problem takes the fused two-tiles-per-CTA scoring kernel (its grid
    # barrier), several the persistent one (its per-problem counters).
    import rank_decode_attention_b200 as s4r
    batch = make_batch(W1, lengths=lengths, top_k=256, tag="timeout")
    ws = workspace_for(batch)
    s4r.s4r_debug_waits(2_000_000, True)          # ~1 ms limit, grid barrier never completes
    try:
        res = run_gpu(batch, workspace=ws)
    finally:
        s4r.s4r_debug_waits(0, False)
    assert res["status"] == s4r.S4R_ERR_TIMEOUT
    assert torch.isfinite(res["out"]).all()
    idx = res["idx"].numpy()
    for b, L in enumerate(batch.lengths):
        got = idx[b][idx[b] >= 0]
        assert np.all(np.diff(got) > 0) and (got.size == 0 or got.max() < 4 + L)
    # The status is sticky until cleared; then the same workspace serves a
    # call whose results match the oracle.
    assert s4r.s4r_read_device_status(ws) == s4r.S4R_ERR_TIMEOUT
    s4r.s4r_clear_device_status(ws)
    res = run_gpu(batch, workspace=ws)
    assert res["status"] == 0
    check_batch(batch, res)


def test_cache_beyond_the_cluster_top_k():
    """More candidates than the 8-CTA cluster select holds (8 x 16384 keys):
    the single-CTA radix select over keys in global memory takes the top-k
    (small-model shape with fp32 storage, so the inputs stay light)."""
    W0 = synth.WORKLOADS[0]
    batch = make_batch(W0, lengths=[140000], top_k=1024, local_window=64, tag="beyond-cluster")
    res = run_gpu(batch)
    assert res["status"] == 0
    check_batch(batch, res)


def test_avg_pooling_kernel7():
    _run(make_batch(W1, lengths=[2500, 900, 40], top_k=128, pool_kernel=7, pool_mode=1, tag="avgpool"))


def test_avg_pooling_exact_ties_from_repeated_rows():
    # Key rows repeat three vectors, so the scores take three values and the
    # pooled means of the interior windows repeat with period three: exact
    # ties among thousands of candidates, decided by position.
    batch = make_batch(W1, lengths=[9000], top_k=1500, pool_kernel=7, pool_mode=1, tag="avgtie")
    g = torch.Generator().manual_seed(9)
    pats = synth.store(torch.randn(3, batch.coeff_k.shape[2], generator=g, dtype=torch.float64) * 0.5, "bf16")
    batch.coeff_k[0, :9000] = pats[torch.arange(9000) % 3]
    res = run_gpu(batch)
    assert res["status"] == 0
    check_batch(batch, res)
    _, idx_ref, _ = oracle.decode_step(batch.oracle_problem(0))
    assert np.array_equal(res["idx"][0].numpy(), idx_ref)
