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
