"""s4r_decode_step_noalloc: the decode step on the library's fixed
per-device scratch array, for callers that cannot provide a workspace.

Its results must match s4r_decode_step (the workspace entry point) within the
decode comparators, on two calls in a row (the second call reuses the shared
scratch the first one left behind).  The file is named to be collected last,
so it also runs after every other GPU test has used the device.
"""
import dataclasses

import pytest
import torch

import synth
from problems import OUT_TOL, SCORE_REL_TOL, make_batch, run_gpu

W0, W1 = synth.WORKLOADS[0], synth.WORKLOADS[1]


def _noalloc_call(batch, expect=0):
    """One s4r_decode_step_noalloc call on the batch (no workspace passed)."""
    import rank_decode_attention_b200 as s4r
    dev = lambda t: t.to("cuda").contiguous()
    q, ck, cv, bk, bv, sk, sv = map(dev, (batch.q, batch.coeff_k, batch.coeff_v, batch.basis_k,
                                          batch.basis_v, batch.sink_k, batch.sink_v))
    B, W, Hq, dh = batch.q.shape
    lengths = torch.tensor(batch.lengths, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hq, dh), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((B, max(batch.top_k, 1)), -7, dtype=torch.int32, device="cuda")
    scores = torch.full((B, batch.cache_rows), float("nan"), device="cuda")
    a = s4r.decode_args(q=q, coeff_k=ck, coeff_v=cv, basis_k=bk, basis_v=bv, sink_k=sk, sink_v=sv,
                        lengths=lengths, n_heads_kv=batch.n_heads_kv, local_window=batch.local_window,
                        top_k=batch.top_k, out=out, idx=idx, scores=scores,
                        pool_kernel=batch.pool_kernel, pool_mode=batch.pool_mode, row_mode=batch.row_mode)
    assert a.workspace is None
    s4r.s4r_decode_step_noalloc(a)
    assert s4r.s4r_read_device_status(None) == expect
    return dict(out=out.cpu(), idx=idx[:, :batch.top_k].cpu(), scores=scores.cpu())


def _noalloc_twice(batch):
    return [_noalloc_call(batch) for _ in range(2)]


def _compare(batch, ref, got):
    max_abs, mean_abs = OUT_TOL[batch.dtype]
    d = (got["out"].double() - ref["out"].double()).abs()
    assert torch.isfinite(got["out"]).all()
    assert d.max().item() <= max_abs and d.mean().item() <= mean_abs
    assert torch.equal(got["idx"], ref["idx"])
    for b, L in enumerate(batch.lengths):
        r, g = ref["scores"][b, :L].double(), got["scores"][b, :L].double()
        assert (g - r).abs().max().item() <= SCORE_REL_TOL[batch.dtype] * r.abs().max().item()


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["bf16-ragged", "f32", "bf16-pooled-per-head"])
def test_noalloc_matches_workspace_entry_point_twice(case):
    if case == "bf16-ragged":
        batch = make_batch(W1, lengths=[5003, 777, 130], top_k=256, tag="noalloc")
    elif case == "f32":
        batch = make_batch(W0, lengths=[2044], tag="noalloc")
    else:
        batch = make_batch(W1, lengths=[3001, 1500], top_k=200, query_window=4, row_mode=1,
                           pool_kernel=7, tag="noalloc-ph")
    ref = run_gpu(batch)
    assert ref["status"] == 0
    first, second = _noalloc_twice(batch)
    _compare(batch, ref, first)
    _compare(batch, ref, second)


@pytest.mark.gpu
def test_noalloc_device_status_goes_to_the_library_word_and_clears():
    # A length beyond the cache capacity is a condition only the device sees:
    # the call records it in the scratch array's status word, which the entry
    # point folds into the library-wide word and zeroes.  After clearing that
    # word, a clean call reports OK again and matches the workspace entry point.
    import rank_decode_attention_b200 as s4r
    s4r.s4r_clear_device_status(None)
    batch = make_batch(W1, lengths=[300, 200], top_k=16, tag="noalloc-bad")
    bad = dataclasses.replace(batch, lengths=[300, 10 ** 6])
    res = _noalloc_call(bad, expect=s4r.S4R_ERR_DEVICE)
    assert torch.isfinite(res["out"]).all()
    assert (res["idx"][1] == -1).all()
    s4r.s4r_clear_device_status(None)
    assert s4r.s4r_read_device_status(None) == s4r.S4R_OK
    ref = run_gpu(batch)
    assert ref["status"] == 0
    _compare(batch, ref, _noalloc_call(batch))


@pytest.mark.gpu
def test_noalloc_calls_of_different_shapes_back_to_back():
    # Calls with other shapes reuse the shared array in between; each must
    # still match the workspace entry point.
    import rank_decode_attention_b200 as s4r
    s4r.s4r_clear_device_status(None)
    a = make_batch(W1, lengths=[5003, 777, 130], top_k=256, tag="noalloc-a")
    b = make_batch(W0, lengths=[2044], tag="noalloc-b")
    c = make_batch(W1, lengths=[1500], top_k=64, pool_kernel=7, pool_mode=1, tag="noalloc-c")
    refs = {id(x): run_gpu(x) for x in (a, b, c)}
    for x in (a, b, c, a, c, b):
        _compare(x, refs[id(x)], _noalloc_call(x))


def test_noalloc_rejects_shapes_beyond_the_scratch():
    """Rejected on the host before any device work (runs without a GPU)."""
    import rank_decode_attention_b200 as s4r
    from rank_decode_attention_b200 import build as s4r_build
    s4r_build.build()
    a = s4r.DecodeArgs()
    a.batch, a.n_heads_q, a.n_heads_kv, a.head_dim, a.rank_k, a.rank_v = 4, 32, 8, 128, 256, 256
    a.n_sink, a.local_window, a.top_k, a.query_window, a.pool_kernel = 4, 128, 1024, 16, 1
    a.dtype, a.cache_rows = s4r.S4R_BF16, 1 << 20
    assert s4r.s4r_decode_workspace_bytes(a) > (4 << 20)
    rc = s4r.lib().s4r_decode_step_noalloc(a, None)
    assert rc == s4r.S4R_ERR_UNSUPPORTED
    assert "scratch" in s4r.s4r_last_error()
