"""GPU parity of the prefill bases (s4r_build_basis) against the fp64 oracle.

The bases are the top-r right singular vectors of the 7:3 sample (Eqs. 1-2).
Where the spectrum has distinct values the subspace they span is unique, so
the comparison is on the projector B B^T; singular values, orthonormality,
the sign convention and the columns of isolated singular values are compared
too, and the storage-type output must be the fp64 result rounded (fp64 ->
fp32 -> storage type, nearest even).

Tolerances come from the arithmetic: both sides work in fp64 and the Jacobi
rotations stop once every off-diagonal entry is below 1e-12 of the geometric
mean of its diagonal pair, so a direction near the rank cut moves by about
1e-12 times the Gram's relative spectral range over the gap; 1e-9 plus that
bound covers the projector.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import basis as obasis
import rank_decode_attention_b200 as s4r

pytestmark = pytest.mark.gpu


def _states(P, L_max, D, true_rank, seed, dtype):
    X = torch.zeros(P, L_max, D, dtype=torch.float64)
    for p in range(P):
        X[p] = synth.states(L_max, D, true_rank, 4, 8, False, synth.seed_of("basis", seed, p))
    return synth.store(X, dtype)


def _run(states, lengths, rank, n_sink, n_sample):
    dev = "cuda"
    P, _, D = states.shape
    st = states.to(dev)
    ln = torch.tensor(lengths, dtype=torch.int32, device=dev)
    out = torch.empty(P, D, rank, dtype=states.dtype, device=dev)
    f64 = torch.empty(P, D, rank, dtype=torch.float64, device=dev)
    sig = torch.empty(P, rank, dtype=torch.float64, device=dev)
    a = s4r.basis_args(states=st, lengths=ln, rank=rank, n_sink=n_sink, n_sample=n_sample)
    nb = s4r.s4r_basis_workspace_bytes(a)
    assert nb > 0
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    s4r.s4r_workspace_init(ws)
    a = s4r.basis_args(states=st, lengths=ln, rank=rank, n_sink=n_sink, n_sample=n_sample, basis_out=out,
                       basis_f64=f64, sigma=sig, workspace=ws)
    s4r.s4r_build_basis(a)
    status = s4r.s4r_read_device_status(ws)
    return status, out.cpu(), f64.cpu().numpy(), sig.cpu().numpy()


def _check_problem(X, L, s, T, r, B, sig, out_row):
    Bo, so, rows = obasis.build_basis(X, L, s, T, r)
    n = len(rows)
    full = min(n, X.shape[1])
    _, s_all, _ = obasis.build_basis(X, L, s, T, full)
    # singular values
    assert np.abs(sig - so).max() <= 1e-11 * so[0]
    # orthonormal, signed
    assert np.abs(B.T @ B - np.eye(r)).max() < 1e-10
    for k in range(r):
        d = int(np.argmax(np.abs(B[:, k])))
        assert B[d, k] > 0
    # projector
    lam = s_all ** 2
    rel_gap = (lam[r - 1] - lam[r]) / lam[0] if r < full else 1.0
    tol = 1e-9 + 1e-12 / rel_gap
    assert np.abs(B @ B.T - Bo @ Bo.T).max() <= tol, (np.abs(B @ B.T - Bo @ Bo.T).max(), tol)
    # columns of isolated singular values
    for k in range(r):
        lo = lam[k - 1] - lam[k] if k > 0 else np.inf
        hi = lam[k] - lam[k + 1] if k + 1 < full else np.inf
        gap = min(lo, hi) / lam[0]
        if gap > 1e-6:
            assert np.abs(B[:, k] - Bo[:, k]).max() <= 1e-9 + 1e-12 / gap, k
    # storage type = fp64 rounded through fp32
    ref = torch.from_numpy(B).to(torch.float32).to(out_row.dtype)
    assert torch.equal(out_row.view(torch.int16) if out_row.dtype == torch.bfloat16 else out_row,
                       ref.view(torch.int16) if ref.dtype == torch.bfloat16 else ref)


CASES = [
    # (name, dtype, P, L list, D, true_rank, r, s, T'): Gram of the rows when T' <= D'
    ("llama-32k-rows", synth.BF16, 2, [32768, 32768], 1024, 64, 192, 4, 256),
    ("batched-8k-ragged", synth.BF16, 3, [8192, 5000, 700], 1024, 128, 128, 4, 512),
    ("short-prompt-padded", synth.BF16, 2, [150, 2000], 256, 32, 64, 4, 256),
    ("odd-sizes", synth.F32, 2, [900, 611], 72, 16, 20, 3, 37),
    ("sample-equals-rank", synth.F32, 1, [68], 128, 16, 64, 4, 64),
    # Gram of the columns when T' > D'
    ("tiny-columns", synth.F32, 2, [2048, 1500], 128, 32, 32, 4, 256),
    ("full-width-columns", synth.BF16, 1, [4096], 64, 16, 64, 4, 300),
    # the largest Gram matrix: D' = 1024 columns, 64 index blocks, 63 block rounds per sweep
    ("max-gram-columns", synth.BF16, 1, [4096], 1024, 64, 256, 4, 2048),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_basis_matches_oracle(case):
    name, dtype, P, Ls, D, true_rank, r, s, T = case
    states = _states(P, max(Ls), D, true_rank, name, dtype)
    status, out, B, sig = _run(states, Ls, r, s, T)
    assert status == s4r.S4R_OK
    Xd = states.to(torch.float64).numpy()
    for p in range(P):
        _check_problem(Xd[p], Ls[p], s, T, r, B[p], sig[p], out[p])


def test_basis_flags_a_sample_shorter_than_the_rank():
    states = _states(2, 600, 64, 16, "short", synth.F32)
    status, *_ = _run(states, [600, 4 + 10], 16, 4, 64)     # second problem: 10 rows < rank 16
    assert status == s4r.S4R_ERR_DEVICE


def test_basis_flags_a_length_beyond_the_rows():
    states = _states(1, 300, 64, 16, "long", synth.F32)
    status, *_ = _run(states, [301], 16, 4, 64)
    assert status == s4r.S4R_ERR_DEVICE


def test_basis_feeds_the_encoder():
    """The bf16 basis from the GPU, used by s4r_encode, gives coefficients
    that rebuild each state's projection onto the basis (Eq. 3, then Eq. 16)."""
    states = _states(1, 4096, 256, 32, "encode", synth.BF16)
    status, out, B, _ = _run(states, [4096], 32, 4, 128)
    assert status == s4r.S4R_OK
    X = states[0].to(torch.float64).numpy()
    P = B[0] @ B[0].T
    Xs = X[4:]
    c = torch.empty(4092, 32, dtype=torch.bfloat16, device="cuda")
    s4r.s4r_encode(states[0, 4:].to("cuda"), out[0].to("cuda").contiguous(), c)
    rec = c.double().cpu().numpy() @ out[0].double().numpy().T
    err = np.linalg.norm(rec - Xs @ P) / np.linalg.norm(Xs @ P)
    assert err < 2e-2
