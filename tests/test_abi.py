"""Host-side checks of the C ABI that need no GPU: every symbol the header
declares is exported, the ctypes structures match the C layout, and argument
errors are reported before anything is enqueued (these calls never reach the
CUDA runtime)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import rank_decode_attention_b200 as s4r
from rank_decode_attention_b200 import build as s4r_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s4r.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    s4r_build.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(s4r_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_expected_entry_points():
    assert set(declared_functions()) >= {"s4r_encode", "s4r_append", "s4r_decode_step",
                                         "s4r_decode_workspace_bytes", "s4r_workspace_init",
                                         "s4r_reconstruct", "s4r_read_device_status",
                                         "s4r_clear_device_status", "s4r_status_string",
                                         "s4r_version"}


def test_library_exports_every_declared_symbol():
    lib = s4r.lib()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", s4r.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (s4r_\w+)", out))
    assert set(declared_functions()) <= exported
    assert set(s4r.SIGNATURES) == set(declared_functions())


def test_struct_layouts_match_c():
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "s4r.h"
#define F(T, m) printf(#T " " #m " %zu\n", offsetof(T, m));
int main(void) {
  printf("s4r_decode_args size %zu\n", sizeof(s4r_decode_args));
  printf("s4r_append_args size %zu\n", sizeof(s4r_append_args));
  F(s4r_decode_args, cache_rows) F(s4r_decode_args, lengths) F(s4r_decode_args, out)
  F(s4r_decode_args, workspace) F(s4r_decode_args, workspace_bytes) F(s4r_decode_args, dtype)
  F(s4r_decode_args, pool_mode) F(s4r_decode_args, row_mode)
  F(s4r_append_args, cache_rows) F(s4r_append_args, lengths) F(s4r_append_args, status_workspace)
  printf("s4r_basis_args size %zu\n", sizeof(s4r_basis_args));
  F(s4r_basis_args, dtype) F(s4r_basis_args, state_rows) F(s4r_basis_args, lengths) F(s4r_basis_args, sigma)
  F(s4r_basis_args, workspace) F(s4r_basis_args, workspace_bytes)
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(src, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    c = {tuple(l.split()[:2]): int(l.split()[2]) for l in lines if l}
    assert c[("s4r_decode_args", "size")] == ctypes.sizeof(s4r.DecodeArgs)
    assert c[("s4r_append_args", "size")] == ctypes.sizeof(s4r.AppendArgs)
    assert c[("s4r_basis_args", "size")] == ctypes.sizeof(s4r.BasisArgs)
    for (T, m), off in c.items():
        if m == "size":
            continue
        cls = {"s4r_decode_args": s4r.DecodeArgs, "s4r_append_args": s4r.AppendArgs,
               "s4r_basis_args": s4r.BasisArgs}[T]
        assert getattr(cls, m).offset == off, (T, m)


def good_args(**over):
    kw = dict(batch=2, n_heads_q=32, n_heads_kv=8, head_dim=128, rank_k=192, rank_v=192, n_sink=4,
              local_window=128, top_k=1024, query_window=16, pool_kernel=1, row_mode=0, dtype=1,
              cache_rows=32768, lengths=0x1000, q=0x2000, coeff_k=0x3000, coeff_v=0x4000,
              basis_k=0x5000, basis_v=0x6000, sink_k=0x7000, sink_v=0x8000, out=0x9000,
              idx=0xa000, scores=None, workspace=0xb000, workspace_bytes=0)
    kw.update(over)
    a = s4r.DecodeArgs()
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_workspace_bytes_and_shape_validation():
    n = s4r.s4r_decode_workspace_bytes(good_args())
    assert n > 0 and n % 256 == 0
    assert s4r.s4r_decode_workspace_bytes(good_args(cache_rows=65536)) > n
    assert s4r.s4r_decode_workspace_bytes(good_args(pool_kernel=7)) > n
    for bad in (dict(n_heads_q=30), dict(rank_k=0), dict(pool_kernel=4), dict(dtype=9),
                dict(row_mode=3), dict(query_window=0), dict(top_k=-1), dict(head_dim=100),
                dict(rank_v=264), dict(n_heads_kv=16, head_dim=128), dict(pool_mode=2)):
        assert s4r.s4r_decode_workspace_bytes(good_args(**bad)) == 0, bad


def call_decode(a):
    return s4r.lib().s4r_decode_step(ctypes.byref(a), None)


def test_decode_argument_errors_are_reported_before_launch():
    ok = s4r.s4r_decode_workspace_bytes(good_args())
    assert call_decode(good_args(n_heads_q=30)) == s4r.S4R_ERR_INVALID_ARG
    assert call_decode(good_args(rank_k=12)) == s4r.S4R_ERR_UNSUPPORTED
    assert call_decode(good_args(query_window=160)) == s4r.S4R_ERR_UNSUPPORTED   # 640 scoring rows
    assert call_decode(good_args(query_window=16, row_mode=1, workspace_bytes=0)) == s4r.S4R_ERR_WORKSPACE   # 512 per-head rows
    assert call_decode(good_args(q=0x2004, workspace_bytes=ok)) == s4r.S4R_ERR_INVALID_ARG
    assert call_decode(good_args(out=None, workspace_bytes=ok)) == s4r.S4R_ERR_INVALID_ARG
    assert call_decode(good_args(sink_k=None, workspace_bytes=ok)) == s4r.S4R_ERR_INVALID_ARG
    assert call_decode(good_args(workspace_bytes=ok - 256)) == s4r.S4R_ERR_WORKSPACE
    assert call_decode(good_args(workspace=None, workspace_bytes=ok)) == s4r.S4R_ERR_WORKSPACE
    assert call_decode(good_args(batch=0)) == s4r.S4R_OK          # empty batch: nothing to do
    assert s4r.lib().s4r_decode_step(None, None) == s4r.S4R_ERR_INVALID_ARG


def test_encode_and_reconstruct_argument_errors():
    L = s4r.lib()
    assert L.s4r_encode(0x1000, 0, 1024, 0x2000, 1024, 256, 0x3000, 256, 1, None) == s4r.S4R_OK
    assert L.s4r_encode(0x1008, 5, 1024, 0x2000, 1024, 256, 0x3000, 256, 1, None) == s4r.S4R_ERR_INVALID_ARG
    assert L.s4r_encode(0x1000, 5, 1000, 0x2000, 1024, 256, 0x3000, 256, 1, None) == s4r.S4R_ERR_INVALID_ARG
    assert L.s4r_encode(0x1000, 5, 1028, 0x2000, 1028, 256, 0x3000, 256, 1, None) == s4r.S4R_ERR_INVALID_ARG
    assert L.s4r_encode(0x1000, 5, 2048, 0x2000, 2048, 256, 0x3000, 256, 1, None) == s4r.S4R_ERR_UNSUPPORTED
    assert L.s4r_encode(0x1000, 5, 1024, 0x2000, 1024, 256, 0x3000, 256, 7, None) == s4r.S4R_ERR_INVALID_ARG
    assert L.s4r_reconstruct(0x1000, 10, 0x2000, 1024, 12, 0x3000, 4, 0x4000, 1, None) == s4r.S4R_ERR_UNSUPPORTED
    assert L.s4r_reconstruct(0x1000, 10, 0x2000, 1024, 16, 0x3000, 0, 0x4000, 1, None) == s4r.S4R_OK


def test_status_strings():
    names = {s4r.s4r_status_string(c) for c in range(7)}
    assert len(names) == 7
    assert s4r.s4r_status_string(99) == "unknown status"
    assert s4r.s4r_version() >= 100


def basis_good(**over):
    kw = dict(n_problems=4, d_model=1024, rank=192, n_sink=4, n_sample=256, dtype=1, state_rows=32768,
              lengths=0x1000, states=0x2000, basis_out=0x3000, basis_f64=None, sigma=None,
              workspace=0x4000, workspace_bytes=0)
    kw.update(over)
    a = s4r.BasisArgs()
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_basis_workspace_bytes_and_validation():
    n = s4r.s4r_basis_workspace_bytes(basis_good())
    # Gram of the 256 sampled rows and its eigenvectors per problem, two buffers of the 32 x 32
    # rotations of its 8 block pairs, plus the fp64 columns, in fp64
    assert n >= 4 * (2 * 256 * 256 + 2 * 8 * 32 * 32 + 1024 * 192) * 8 and n % 256 == 0
    # more samples than D': the Gram of the 1024 columns instead
    assert s4r.s4r_basis_workspace_bytes(basis_good(n_sample=2048)) >= 4 * 2 * 1024 * 1024 * 8
    for bad in (dict(rank=0), dict(rank=257, n_sample=300), dict(rank=300, n_sample=200), dict(dtype=7),
                dict(d_model=0), dict(n_sample=0), dict(n_problems=-1), dict(d_model=2048),
                dict(n_sink=-1), dict(state_rows=-5)):
        assert s4r.s4r_basis_workspace_bytes(basis_good(**bad)) == 0, bad
    lib = s4r.lib()
    assert lib.s4r_build_basis(ctypes.byref(basis_good(rank=300, n_sample=200)), None) == s4r.S4R_ERR_INVALID_ARG
    assert lib.s4r_build_basis(ctypes.byref(basis_good(d_model=2048)), None) == s4r.S4R_ERR_UNSUPPORTED
    assert lib.s4r_build_basis(ctypes.byref(basis_good(states=0x2008)), None) == s4r.S4R_ERR_INVALID_ARG
    assert lib.s4r_build_basis(ctypes.byref(basis_good(basis_out=None)), None) == s4r.S4R_ERR_INVALID_ARG
    assert lib.s4r_build_basis(ctypes.byref(basis_good(workspace_bytes=64)), None) == s4r.S4R_ERR_WORKSPACE
    assert lib.s4r_build_basis(ctypes.byref(basis_good(n_problems=0)), None) == s4r.S4R_OK
