"""Parity of the CUDA decode step against the fp64 oracle, through the C ABI.

Comparators (from the decode path's accuracy contract):
  * selected index sets bit-exact except swaps between candidates whose fp64
    scores are within 1e-6 (relative to the k-th score);
  * out vs the oracle evaluated at the GPU's own index set: bf16 storage
    max-abs 2e-2 / mean-abs 2e-3, fp32 storage 1e-4;
  * latent scores within 5e-6 of the fp64 scores (relative to the largest).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from problems import check_batch, make_batch, run_gpu

pytestmark = pytest.mark.gpu

W0, W1, W2, W3, W4 = (synth.WORKLOADS[i] for i in range(5))


def _run(batch, **kw):
    res = run_gpu(batch)
    assert res["status"] == 0, f"device status {res['status']}"
    return check_batch(batch, res, **kw)


def test_tiny_f32_workload():
    # prompt 2048 tokens, 4 sinks -> 2044 coefficient rows
    _run(make_batch(W0, lengths=[2048 - 4]))


@pytest.mark.parametrize("lengths", [[5003, 777, 130], [64 * 7 + 1], [1000, 2000]])
def test_bf16_multi_tile_ragged(lengths):
    _run(make_batch(W1, lengths=lengths, top_k=256, tag="ragged"))


def test_per_head_rows():
    _run(make_batch(W1, lengths=[3001, 1500], top_k=200, query_window=4, row_mode=1, tag="ph"))


def test_pooling_kernel7():
    _run(make_batch(W1, lengths=[2500, 900], top_k=128, pool_kernel=7, tag="pool"))


def test_asymmetric_ranks():
    _run(make_batch(W1, lengths=[1800, 2600], rank_k=128, rank_v=192, top_k=100, tag="asym"))


def test_no_sinks_and_small_windows():
    _run(make_batch(W1, lengths=[700, 65], n_sink=0, local_window=8, top_k=40,
                    query_window=2, tag="nosink"))


@pytest.mark.parametrize("lengths,k,w", [([0, 3, 50], 16, 64), ([10, 100], 0, 32),
                                          ([64, 65, 66], 8, 64), ([300], 300, 0)])
def test_edge_lengths(lengths, k, w):
    _run(make_batch(W1, lengths=lengths, top_k=k, local_window=w, tag="edge",
                    cache_rows=max(lengths) + 5))


def test_f32_storage_bigger_shape():
    w = synth.Workload(**{**W1.__dict__, "dtype": "f32"})
    _run(make_batch(w, lengths=[3000], top_k=300, tag="f32big"))


def test_llama_shape_L32k_one_layer():
    """Full-size Llama-3-8B-shaped problem (L = 32768, r = 192), two steps."""
    for step in (0, 1):
        _run(make_batch(W1, lengths=[32768 - 4], layer=3, step=step))


def test_llama_shape_L32k_two_problems_one_call():
    """Two full-size 32K problems in one call (the shape of the
    all-layers-in-one-call variant): the row-split attention with 16-CTA
    clusters at full size."""
    _run(make_batch(W1, lengths=[32768 - 4, 32768 - 4], layer=5))


def test_batched_16x8k():
    _run(make_batch(W2, lengths=[8192 - 4] * 16, layer=1))


def test_long_context_128k_one_layer():
    _run(make_batch(W3, lengths=[131072 - 4], layer=2))


def test_ragged_eight_sequences():
    lens = [L - 4 for L in synth.lengths(W4)]
    _run(make_batch(W4, lengths=lens))


def test_device_status_on_bad_length():
    import rank_decode_attention_b200 as s4r
    batch = make_batch(W1, lengths=[300, 200], top_k=16, tag="bad")
    batch.lengths = [300, 10**6]          # second length beyond the cache capacity
    res = run_gpu(batch, want_scores=False)
    assert res["status"] == s4r.S4R_ERR_DEVICE
    assert torch.isfinite(res["out"]).all()
    assert (res["idx"][1] == -1).all()


def _run_exact_idx(batch):
    """Run the batch and also require the index sets to equal the oracle's
    exactly: these cases are built so that ties are decided by position."""
    res = run_gpu(batch)
    assert res["status"] == 0, f"device status {res['status']}"
    check_batch(batch, res)
    for b in range(batch.batch):
        _, idx_ref, _ = oracle.decode_step(batch.oracle_problem(b))
        assert np.array_equal(res["idx"][b].numpy(), idx_ref), f"problem {b}: tie order differs"
    return res


def test_all_scores_tied_take_lowest_positions():
    # Zero key coefficients: every logit is 0, every score equal, so the top-k
    # is the k lowest candidate positions (and every rank's candidate buffer
    # overflows, which sends the cluster select to its exact path).
    batch = make_batch(W1, lengths=[20000, 9000], top_k=512, tag="tied")
    batch.coeff_k.zero_()
    res = _run_exact_idx(batch)
    for b in range(2):
        assert np.array_equal(res["idx"][b].numpy(), 4 + np.arange(512))


@pytest.mark.parametrize("top_k", [1000, 4000])
def test_three_distinct_rows_tie_across_ranks(top_k):
    # Key rows repeat three vectors, so the scores take three values and the
    # threshold value is shared by thousands of keys spread over the cluster.
    batch = make_batch(W1, lengths=[9000], top_k=top_k, tag="three")
    g = torch.Generator().manual_seed(7)
    pats = synth.store(torch.randn(3, batch.coeff_k.shape[2], generator=g, dtype=torch.float64) * 0.5, "bf16")
    batch.coeff_k[0, :9000] = pats[torch.arange(9000) % 3]
    _run_exact_idx(batch)


@pytest.mark.parametrize("rank_k,rank_v", [(136, 200), (200, 136), (64, 72)])
def test_ranks_off_the_tensor_core_tiles(rank_k, rank_v):
    # Ranks that are not multiples of 16 take the CUDA-core logits / value-sum
    # paths of the attention kernel (and odd 64-column blocks of the scoring).
    _run(make_batch(W1, lengths=[3100, 1700], rank_k=rank_k, rank_v=rank_v, top_k=300, tag="oddrank"))


def test_many_selected_rows_take_several_chunks():
    # k + w large enough that a CTA of the row-split attention cluster (two
    # problems per call) stages its rows in more than one pass (rank 256
    # shrinks the staging capacity); the single problem takes the per-group
    # kernel with the same selection size.
    _run(make_batch(W3, lengths=[40000, 36000], top_k=3000, local_window=512, tag="chunks"))
    _run(make_batch(W3, lengths=[40000], top_k=3000, local_window=512, tag="chunks"))


def test_ragged_append_then_decode_steps():
    """The ragged append workload over several steps: each step first appends
    one encoded token per sequence (s4r_append on the device caches), then
    decodes.  Appended rows match the fp64 encode within one bf16 ulp; each
    decode is compared with the oracle run on the GPU's appended cache."""
    import dataclasses
    import rank_decode_attention_b200 as s4r
    from test_gpu_encode import check_encode
    lens = [L - 4 for L in synth.lengths(W4)]
    batch = make_batch(W4, lengths=lens, cache_rows=max(lens) + 8, tag="append")
    B, D = batch.batch, batch.basis_k.shape[1]
    ck, cv = batch.coeff_k.cuda(), batch.coeff_v.cuda()
    bk, bv = batch.basis_k.cuda(), batch.basis_v.cuda()
    lengths = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    s4r.s4r_workspace_init(ws)
    g = torch.Generator().manual_seed(21)
    for step in range(3):
        new_k = synth.store(torch.randn(B, D, generator=g, dtype=torch.float64), "bf16")
        new_v = synth.store(torch.randn(B, D, generator=g, dtype=torch.float64), "bf16")
        s4r.s4r_append(state_k=new_k.cuda(), state_v=new_v.cuda(), basis_k=bk, basis_v=bv,
                       coeff_k=ck, coeff_v=cv, lengths=lengths, status_workspace=ws)
        assert s4r.s4r_read_device_status(ws) == s4r.S4R_OK
        Ls = lengths.cpu().tolist()
        assert Ls == [L + step + 1 for L in lens]
        ck_h, cv_h = ck.cpu(), cv.cpu()
        for b in range(B):
            row = Ls[b] - 1
            check_encode(new_k[b:b + 1], batch.basis_k[b], ck_h[b, row:row + 1], "bf16")
            check_encode(new_v[b:b + 1], batch.basis_v[b], cv_h[b, row:row + 1], "bf16")
        q = synth.store(torch.randn(batch.q.shape, generator=g, dtype=torch.float64), "bf16")
        step_batch = dataclasses.replace(batch, q=q, coeff_k=ck_h, coeff_v=cv_h, lengths=Ls)
        _run(step_batch)


def test_many_small_problems_single_cta_clusters():
    # G = 1 (as many query heads as kv heads) and 40 problems: one head per
    # CTA of each problem's attention cluster, and more clusters than fit on
    # the device at once.
    w = synth.Workload(**{**W1.__dict__, "n_heads_q": 8})
    _run(make_batch(w, lengths=[600 + 37 * i for i in range(40)], top_k=64, local_window=32, tag="g1"))
