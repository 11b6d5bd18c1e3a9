"""Parity of encode (C = S . B), append and explicit rebuild against the oracle.

Encode comparator: |gpu - exact| <= one storage ulp at |exact| plus the fp32
accumulation bound 2^-20 * sum_d |S_d B_dj| (bf16), or 1e-5 relative to that
sum (fp32 storage).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_encode(S: torch.Tensor, B: torch.Tensor, C_gpu: torch.Tensor, dtype: str):
    Sd, Bd = S.double().numpy(), B.double().numpy()
    exact = oracle.encode(Sd, Bd)
    scale = np.abs(Sd) @ np.abs(Bd)
    got = C_gpu.double().numpy()
    if dtype == "bf16":
        bound = bf16_ulp(exact) + 2.0 ** -20 * scale
    else:
        bound = 1e-5 * scale + 1e-30
    bad = np.abs(got - exact) > bound
    assert not bad.any(), f"{bad.sum()} coefficients off, worst {np.abs(got - exact)[bad].max():.3e}"


@pytest.mark.parametrize("dtype,n,d,r", [("bf16", 3000, 1024, 256), ("bf16", 129, 1024, 192),
                                         ("bf16", 1, 128, 32), ("f32", 700, 128, 32),
                                         ("bf16", 4096, 1024, 128)])
def test_encode_matches_oracle(dtype, n, d, r):
    import rank_decode_attention_b200 as s4r
    g = torch.Generator().manual_seed(n * 7 + r)
    S = synth.store(torch.randn(n, d, generator=g, dtype=torch.float64), dtype)
    B = synth.store(torch.randn(d, r, generator=g, dtype=torch.float64) / d ** 0.5, dtype)
    C = torch.empty(n, r, dtype=S.dtype, device="cuda")
    s4r.s4r_encode(S.cuda(), B.cuda(), C)
    torch.cuda.synchronize()
    check_encode(S, B, C.cpu(), dtype)


@pytest.mark.parametrize("dtype,n,d,r", [("bf16", 3000, 1024, 256), ("bf16", 129, 1024, 192),
                                         ("bf16", 1, 128, 32), ("f32", 300, 128, 32), ("bf16", 500, 256, 48)])
def test_encode2_matches_oracle_for_both_problems(dtype, n, d, r):
    """The two-problem launch (K and V halves, each with its own basis) gives
    each half exactly the oracle's encode; tile counts that are not a multiple
    of the grid put both problems' tiles on one CTA."""
    import rank_decode_attention_b200 as s4r
    g = torch.Generator().manual_seed(n * 11 + r)
    S = [synth.store(torch.randn(n, d, generator=g, dtype=torch.float64), dtype) for _ in range(2)]
    B = [synth.store(torch.randn(d, r, generator=g, dtype=torch.float64) / d ** 0.5, dtype) for _ in range(2)]
    C = [torch.full((n, r), float("nan"), dtype=S[0].dtype, device="cuda") for _ in range(2)]
    s4r.s4r_encode2([x.cuda() for x in S], [x.cuda() for x in B], C)
    torch.cuda.synchronize()
    for p in range(2):
        check_encode(S[p], B[p], C[p].cpu(), dtype)


def test_encode_strided_rows():
    import rank_decode_attention_b200 as s4r
    g = torch.Generator().manual_seed(5)
    big = synth.store(torch.randn(300, 1040, generator=g, dtype=torch.float64), "bf16").cuda()
    S = big[:, :1024]                                   # row stride 1040
    B = synth.store(torch.randn(1024, 64, generator=g, dtype=torch.float64) / 32, "bf16").cuda()
    Cbig = torch.zeros(300, 72, dtype=torch.bfloat16, device="cuda")
    C = Cbig[:, :64]
    s4r.s4r_encode(S, B, C)
    torch.cuda.synchronize()
    check_encode(S.cpu(), B.cpu(), C.cpu(), "bf16")
    assert (Cbig[:, 64:] == 0).all()


def test_append_writes_row_and_bumps_length():
    import rank_decode_attention_b200 as s4r
    g = torch.Generator().manual_seed(11)
    Bn, D, rk, rv, cap = 3, 1024, 256, 192, 50
    st_k = synth.store(torch.randn(Bn, D, generator=g, dtype=torch.float64), "bf16")
    st_v = synth.store(torch.randn(Bn, D, generator=g, dtype=torch.float64), "bf16")
    bk = synth.store(torch.randn(Bn, D, rk, generator=g, dtype=torch.float64) / 32, "bf16")
    bv = synth.store(torch.randn(Bn, D, rv, generator=g, dtype=torch.float64) / 32, "bf16")
    ck = torch.zeros(Bn, cap, rk, dtype=torch.bfloat16, device="cuda")
    cv = torch.zeros(Bn, cap, rv, dtype=torch.bfloat16, device="cuda")
    lengths = torch.tensor([0, 17, cap], dtype=torch.int32, device="cuda")   # last one is full
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    s4r.s4r_workspace_init(ws)
    s4r.s4r_append(state_k=st_k.cuda(), state_v=st_v.cuda(), basis_k=bk.cuda(), basis_v=bv.cuda(),
                   coeff_k=ck, coeff_v=cv, lengths=lengths, status_workspace=ws)
    assert s4r.s4r_read_device_status(ws) == s4r.S4R_ERR_DEVICE      # the full cache was skipped
    assert lengths.cpu().tolist() == [1, 18, cap]
    for b, row in ((0, 0), (1, 17)):
        check_encode(st_k[b:b + 1], bk[b], ck[b, row:row + 1].cpu(), "bf16")
        check_encode(st_v[b:b + 1], bv[b], cv[b, row:row + 1].cpu(), "bf16")
    assert (ck[2] == 0).all() and (cv[2] == 0).all()
    s4r.s4r_clear_device_status(ws)
    assert s4r.s4r_read_device_status(ws) == s4r.S4R_OK


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_reconstruct_matches_oracle(dtype):
    import rank_decode_attention_b200 as s4r
    g = torch.Generator().manual_seed(3)
    C = synth.store(torch.randn(500, 192, generator=g, dtype=torch.float64), dtype)
    B = synth.store(torch.randn(1024, 192, generator=g, dtype=torch.float64) / 14, dtype)
    rows = torch.tensor([0, 499, 17, -1, 500, 250], dtype=torch.int32)
    out = torch.empty(rows.numel(), 1024, device="cuda")
    s4r.s4r_reconstruct(C.cuda(), B.cuda(), rows.cuda(), out)
    torch.cuda.synchronize()
    valid = [0, 1, 2, 5]
    ref = oracle.reconstruct(C.double().numpy()[rows[valid].numpy()], B.double().numpy())
    scale = np.abs(C.double().numpy()[rows[valid].numpy()]) @ np.abs(B.double().numpy()).T
    assert np.all(np.abs(out.cpu().double().numpy()[valid] - ref) <= 1e-5 * scale + 1e-30)
    assert (out[3] == 0).all() and (out[4] == 0).all()
