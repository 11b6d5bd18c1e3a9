"""Parity of the decode step on subsets of every benchmark workload at full
size, through the C ABI against the fp64 oracle (Eqs. 8-18 of the S4R review
page; comparators in tests/problems.py):

  * Llama-3-8B-shaped 32K (L = 32768, r = 192): layers {0, 15, 31} x
    decode steps {0, 1, 2};
  * batched 16 x 8K (r = 128, top-k 512): layers {0, 31} x steps
    {0, 63, 127}, all 16 sequences in one call;
  * long context 128K (r = 256, top-k 2048, window 256): layers {0, 31} x
    all 16 steps;
  * ragged encode + decode (8 sequences, L ~ U[4096, 65536], r = 256): 256
    steps, each appending one encoded token per sequence to the device caches
    (every appended row checked against the fp64 encode) and decoding; the
    decode is checked at steps {0, 1, 127, 255} on the cache the GPU built;
  * the 65536-token bulk prompt encode (D' = 1024, r = 256), every element.

The layers, sequences and query windows come from the seeded generator with
the workloads' own recipe, as in the benchmark.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from problems import check_batch, make_batch, run_gpu
from test_gpu_encode import check_encode

pytestmark = pytest.mark.gpu

W1, W2, W3, W4 = (synth.WORKLOADS[i] for i in (1, 2, 3, 4))


def _run_steps(w, layer, steps, lengths):
    batch, qs = make_batch(w, lengths=lengths, layer=layer, windows=steps, tag=f"subset-l{layer}")
    for t in steps:
        step_batch = dataclasses.replace(batch, q=qs[t])
        res = run_gpu(step_batch)
        assert res["status"] == 0, f"layer {layer} step {t}: device status {res['status']}"
        check_batch(step_batch, res)


@pytest.mark.parametrize("layer", [0, 15, 31])
def test_llama_shape_32k_layer_steps(layer):
    _run_steps(W1, layer, [0, 1, 2], [W1.prompt_len - W1.n_sink])


@pytest.mark.parametrize("layer", [0, 31])
def test_batched_16x8k_layer_steps(layer):
    _run_steps(W2, layer, [0, 63, 127], [W2.prompt_len - W2.n_sink] * W2.batch)


@pytest.mark.parametrize("layer", [0, 31])
def test_long_context_128k_layer_all_steps(layer):
    _run_steps(W3, layer, list(range(W3.steps)), [W3.prompt_len - W3.n_sink])


def test_ragged_append_decode_256_steps():
    import rank_decode_attention_b200 as s4r
    lens = [L - W4.n_sink for L in synth.lengths(W4)]
    n_steps = W4.steps
    check_at = {0, 1, 127, 255}
    batch, qs = make_batch(W4, lengths=lens, cache_rows=max(lens) + n_steps, windows=sorted(check_at),
                           tag="ragged-256")
    B, D = batch.batch, batch.basis_k.shape[1]
    dev = lambda t: t.cuda().contiguous()
    ck, cv, bk, bv = dev(batch.coeff_k), dev(batch.coeff_v), dev(batch.basis_k), dev(batch.basis_v)
    sk, sv = dev(batch.sink_k), dev(batch.sink_v)
    lengths = torch.tensor(lens, dtype=torch.int32, device="cuda")
    g = torch.Generator().manual_seed(4242)
    new_k = synth.store(torch.randn(n_steps, B, D, generator=g, dtype=torch.float64), "bf16")
    new_v = synth.store(torch.randn(n_steps, B, D, generator=g, dtype=torch.float64), "bf16")
    q_any = synth.store(torch.randn(batch.q.shape, generator=g, dtype=torch.float64), "bf16")
    out = torch.empty(B, batch.q.shape[2], batch.q.shape[3], device="cuda")
    idx = torch.empty(B, batch.top_k, dtype=torch.int32, device="cuda")
    kw = dict(coeff_k=ck, coeff_v=cv, basis_k=bk, basis_v=bv, sink_k=sk, sink_v=sv, lengths=lengths,
              n_heads_kv=batch.n_heads_kv, local_window=batch.local_window, top_k=batch.top_k, out=out,
              idx=idx)
    ws = torch.empty(s4r.s4r_decode_workspace_bytes(s4r.decode_args(q=dev(q_any), **kw)), dtype=torch.uint8,
                     device="cuda")
    s4r.s4r_workspace_init(ws)
    nk_dev, nv_dev = dev(new_k), dev(new_v)
    ar = torch.arange(B, device="cuda")
    for t in range(n_steps):
        before = lengths.clone()
        s4r.s4r_append(state_k=nk_dev[t], state_v=nv_dev[t], basis_k=bk, basis_v=bv, coeff_k=ck, coeff_v=cv,
                       lengths=lengths, status_workspace=ws)
        q = dev(qs[t]) if t in check_at else dev(q_any)
        s4r.s4r_decode_step(s4r.decode_args(q=q, workspace=ws, **kw))
        # the row each sequence appended at this step
        got_k, got_v = ck[ar, before.long()].cpu(), cv[ar, before.long()].cpu()
        assert before.cpu().tolist() == [L + t for L in lens]
        for b in range(B):
            check_encode(new_k[t, b:b + 1], batch.basis_k[b], got_k[b:b + 1], "bf16")
            check_encode(new_v[t, b:b + 1], batch.basis_v[b], got_v[b:b + 1], "bf16")
        if t in check_at:
            assert s4r.s4r_read_device_status(ws) == s4r.S4R_OK
            Ls = lengths.cpu().tolist()
            res = dict(out=out.cpu(), idx=idx.cpu(), scores=None, status=0)
            step_batch = dataclasses.replace(batch, q=qs[t], coeff_k=ck.cpu(), coeff_v=cv.cpu(), lengths=Ls)
            check_batch(step_batch, res)
    assert s4r.s4r_read_device_status(ws) == s4r.S4R_OK


def test_per_head_rows_at_the_llama_shape_32k():
    """Per-head scoring rows (W * H_q = 16 * 32 = 512 rows, each head projected
    with its kv group's d_h rows of the key basis) on a full-size 32K layer."""
    batch = make_batch(W1, lengths=[W1.prompt_len - W1.n_sink], layer=5, row_mode=1, tag="per-head-32k")
    res = run_gpu(batch)
    assert res["status"] == 0
    check_batch(batch, res)


def test_bulk_encode_65536_tokens():
    import rank_decode_attention_b200 as s4r
    n, D, r = synth.BULK_ENCODE_TOKENS, 1024, 256
    X = synth.states(n + 4, D, 256, 4, 8, False, synth.seed_of("bulk-encode", "k"))
    rows = synth.sample_rows(n + 4, 4, 256)
    B = synth.store(synth.basis(X, rows, r), "bf16")
    S = synth.store(X[4:], "bf16")
    C = torch.empty(n, r, dtype=torch.bfloat16, device="cuda")
    s4r.s4r_encode(S.cuda(), B.cuda(), C)
    torch.cuda.synchronize()
    check_encode(S, B, C.cpu(), "bf16")
