"""Python binding of libs4r (S4R compressed-KV decode on B200, sm_100a).

Argument marshalling only: every function here fills the C structures of
``include/s4r.h`` from torch tensors (device pointers, sizes read from tensor
shapes) and calls the entry point of the same name in ``libs4r.so``.  All
arithmetic runs in the library's CUDA kernels; there is no Python or CPU
fallback, and a missing or unloadable library raises immediately.

Build the library with ``python -m rank_decode_attention_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libs4r.so")

S4R_OK, S4R_ERR_INVALID_ARG, S4R_ERR_UNSUPPORTED, S4R_ERR_CUDA, S4R_ERR_TIMEOUT, \
    S4R_ERR_DEVICE, S4R_ERR_WORKSPACE = range(7)
S4R_F32, S4R_BF16 = 0, 1
S4R_ROWS_CONCAT, S4R_ROWS_PER_HEAD = 0, 1
S4R_POOL_MAX, S4R_POOL_AVG = 0, 1

_DTYPE = {torch.float32: S4R_F32, torch.bfloat16: S4R_BF16}


class S4RError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = s4r_last_error() if status == S4R_ERR_CUDA else ""
        super().__init__(f"{what}: {s4r_status_string(status)} (status {status})"
                         + (f" -- {detail}" if detail else ""))
        self.status = status


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_heads_q", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("rank_k", ctypes.c_int32), ("rank_v", ctypes.c_int32),
        ("n_sink", ctypes.c_int32), ("local_window", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("query_window", ctypes.c_int32), ("pool_kernel", ctypes.c_int32),
        ("pool_mode", ctypes.c_int32), ("row_mode", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("cache_rows", ctypes.c_int64),
        ("lengths", ctypes.c_void_p), ("q", ctypes.c_void_p),
        ("coeff_k", ctypes.c_void_p), ("coeff_v", ctypes.c_void_p),
        ("basis_k", ctypes.c_void_p), ("basis_v", ctypes.c_void_p),
        ("sink_k", ctypes.c_void_p), ("sink_v", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("idx", ctypes.c_void_p), ("scores", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("profile_events", ctypes.c_void_p * 2),
    ]


class AppendArgs(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("d_model", ctypes.c_int32), ("rank_k", ctypes.c_int32),
        ("rank_v", ctypes.c_int32), ("dtype", ctypes.c_int32), ("cache_rows", ctypes.c_int64),
        ("state_k", ctypes.c_void_p), ("state_v", ctypes.c_void_p),
        ("basis_k", ctypes.c_void_p), ("basis_v", ctypes.c_void_p),
        ("coeff_k", ctypes.c_void_p), ("coeff_v", ctypes.c_void_p),
        ("lengths", ctypes.c_void_p), ("status_workspace", ctypes.c_void_p),
    ]


class BasisArgs(ctypes.Structure):
    _fields_ = [
        ("n_problems", ctypes.c_int32), ("d_model", ctypes.c_int32), ("rank", ctypes.c_int32),
        ("n_sink", ctypes.c_int32), ("n_sample", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("state_rows", ctypes.c_int64),
        ("lengths", ctypes.c_void_p), ("states", ctypes.c_void_p), ("basis_out", ctypes.c_void_p),
        ("basis_f64", ctypes.c_void_p), ("sigma", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


# Exported symbols and their C signatures (restype, argtypes).
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
SIGNATURES = {
    "s4r_encode": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _i32, _vp, _i64, ctypes.c_int, _vp]),
    "s4r_encode2": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _i32, _i32, _vp, _vp, _i64, ctypes.c_int, _vp]),
    "s4r_append": (ctypes.c_int, [ctypes.POINTER(AppendArgs), _vp]),
    "s4r_decode_workspace_bytes": (_sz, [ctypes.POINTER(DecodeArgs)]),
    "s4r_decode_kernel_launches": (_i32, [ctypes.POINTER(DecodeArgs)]),
    "s4r_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "s4r_decode_step": (ctypes.c_int, [ctypes.POINTER(DecodeArgs), _vp]),
    "s4r_decode_step_noalloc": (ctypes.c_int, [ctypes.POINTER(DecodeArgs), _vp]),
    "s4r_basis_workspace_bytes": (_sz, [ctypes.POINTER(BasisArgs)]),
    "s4r_build_basis": (ctypes.c_int, [ctypes.POINTER(BasisArgs), _vp]),
    "s4r_reconstruct": (ctypes.c_int, [_vp, _i64, _vp, _i32, _i32, _vp, _i64, _vp, ctypes.c_int, _vp]),
    "s4r_read_device_status": (ctypes.c_int, [_vp, _vp]),
    "s4r_clear_device_status": (ctypes.c_int, [_vp, _vp]),
    "s4r_debug_waits": (ctypes.c_int, [_i64, _i32]),
    "s4r_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "s4r_version": (_i32, []),
    "s4r_last_error": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libs4r.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m rank_decode_attention_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype, fn.argtypes = res, args
        _lib = h
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> int:
    if status != S4R_OK:
        raise S4RError(status, what)
    return status


def s4r_status_string(status: int) -> str:
    return lib().s4r_status_string(status).decode()


def s4r_last_error() -> str:
    return (lib().s4r_last_error() or b"").decode()


def s4r_version() -> int:
    return int(lib().s4r_version())


def s4r_encode(states: torch.Tensor, basis: torch.Tensor, coeffs: torch.Tensor, stream=None) -> int:
    """coeffs[t] = states[t] . basis (Eq. 3).  states [n][D'] (row stride may
    exceed D'), basis [D'][r], coeffs [n][r] (row stride may exceed r)."""
    n, d = states.shape
    r = basis.shape[1]
    return _check(lib().s4r_encode(_ptr(states), n, states.stride(0), _ptr(basis), d, r,
                                   _ptr(coeffs), coeffs.stride(0), _DTYPE[states.dtype],
                                   _stream(stream)), "s4r_encode")


def s4r_encode2(states, bases, coeffs, stream=None) -> int:
    """coeffs[p][t] = states[p][t] . bases[p] for p = 0, 1 (Eq. 3), one
    launch: two token sets of the same shape and strides with their own
    bases (the K and V halves of a prompt)."""
    s0, s1 = states
    n, d = s0.shape
    r = bases[0].shape[1]
    if s1.shape != s0.shape or s1.stride(0) != s0.stride(0) or coeffs[1].stride(0) != coeffs[0].stride(0):
        raise ValueError("s4r_encode2: both problems need the same shape and strides")
    return _check(lib().s4r_encode2(_ptr(s0), _ptr(s1), n, s0.stride(0), _ptr(bases[0]), _ptr(bases[1]), d, r,
                                    _ptr(coeffs[0]), _ptr(coeffs[1]), coeffs[0].stride(0), _DTYPE[s0.dtype],
                                    _stream(stream)), "s4r_encode2")


def append_args(*, state_k, state_v, basis_k, basis_v, coeff_k, coeff_v, lengths,
                status_workspace=None) -> AppendArgs:
    B, cache_rows, rk = coeff_k.shape
    return AppendArgs(B, basis_k.shape[1], rk, coeff_v.shape[2], _DTYPE[coeff_k.dtype], cache_rows,
                      _ptr(state_k), _ptr(state_v), _ptr(basis_k), _ptr(basis_v), _ptr(coeff_k),
                      _ptr(coeff_v), _ptr(lengths), _ptr(status_workspace))


def s4r_append(stream=None, **kw) -> int:
    """Encode one new token per problem and append it at row lengths[b]."""
    a = append_args(**kw)
    return _check(lib().s4r_append(ctypes.byref(a), _stream(stream)), "s4r_append")


def decode_args(*, q, coeff_k, coeff_v, basis_k, basis_v, sink_k, sink_v, lengths, n_heads_kv,
                local_window, top_k, out=None, idx=None, scores=None, workspace=None,
                workspace_bytes=None, pool_kernel=1, pool_mode=S4R_POOL_MAX,
                row_mode=S4R_ROWS_CONCAT, profile_events=None) -> DecodeArgs:
    """Fill s4r_decode_args from tensors: q [B][W][H_q][d_h], coeff_k/v
    [B][cache_rows][r], basis_k/v [B][D'][r], sink_k/v [B][s][D'],
    lengths [B] int32 (device)."""
    B, W, Hq, dh = q.shape
    cache_rows = coeff_k.shape[1]
    n_sink = sink_k.shape[1] if sink_k is not None else 0
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    a = DecodeArgs(B, Hq, n_heads_kv, dh, coeff_k.shape[2], coeff_v.shape[2], n_sink,
                   local_window, top_k, W, pool_kernel, pool_mode, row_mode, _DTYPE[q.dtype],
                   cache_rows,
                   _ptr(lengths), _ptr(q), _ptr(coeff_k), _ptr(coeff_v), _ptr(basis_k),
                   _ptr(basis_v), _ptr(sink_k), _ptr(sink_v), _ptr(out), _ptr(idx),
                   _ptr(scores), _ptr(workspace), workspace_bytes or 0)
    if profile_events is not None:
        a.profile_events[0] = profile_events[0].cuda_event
        a.profile_events[1] = profile_events[1].cuda_event
    return a


def s4r_decode_kernel_launches(args: DecodeArgs) -> int:
    return int(lib().s4r_decode_kernel_launches(ctypes.byref(args)))


def s4r_decode_workspace_bytes(args: DecodeArgs) -> int:
    return int(lib().s4r_decode_workspace_bytes(ctypes.byref(args)))


def s4r_workspace_init(workspace: torch.Tensor, stream=None) -> int:
    nbytes = workspace.numel() * workspace.element_size()
    return _check(lib().s4r_workspace_init(_ptr(workspace), nbytes, _stream(stream)),
                  "s4r_workspace_init")


def s4r_decode_step(args: DecodeArgs, stream=None) -> int:
    """One decode step for every problem (see include/s4r.h)."""
    return _check(lib().s4r_decode_step(ctypes.byref(args), _stream(stream)), "s4r_decode_step")


def s4r_decode_step_noalloc(args: DecodeArgs, stream=None) -> int:
    """The decode step on the library's fixed per-device scratch array (no
    workspace, nothing allocated; see include/s4r.h for its limits)."""
    return _check(lib().s4r_decode_step_noalloc(ctypes.byref(args), _stream(stream)),
                  "s4r_decode_step_noalloc")


def basis_args(*, states, lengths, rank, n_sink, n_sample, basis_out=None, basis_f64=None, sigma=None,
               workspace=None, workspace_bytes=None) -> BasisArgs:
    """Fill s4r_basis_args: states [P][state_rows][D'] (bf16 or fp32), lengths
    [P] int32 (device), outputs basis_out [P][D'][r] (states' dtype),
    basis_f64 [P][D'][r] float64, sigma [P][r] float64."""
    P, state_rows, d = states.shape
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    return BasisArgs(P, d, rank, n_sink, n_sample, _DTYPE[states.dtype], state_rows, _ptr(lengths),
                     _ptr(states), _ptr(basis_out), _ptr(basis_f64), _ptr(sigma), _ptr(workspace),
                     workspace_bytes or 0)


def s4r_basis_workspace_bytes(args: BasisArgs) -> int:
    return int(lib().s4r_basis_workspace_bytes(ctypes.byref(args)))


def s4r_build_basis(args: BasisArgs, stream=None) -> int:
    """Prefill bases: 7:3 sample, unit-norm rows, top-r right singular
    vectors in fp64 (Eqs. 1-2; see include/s4r.h)."""
    return _check(lib().s4r_build_basis(ctypes.byref(args), _stream(stream)), "s4r_build_basis")


def s4r_reconstruct(coeffs: torch.Tensor, basis: torch.Tensor, rows: torch.Tensor,
                    out: torch.Tensor, stream=None) -> int:
    """out[e] = coeffs[rows[e]] . basis^T in fp32 (Eq. 16)."""
    n_total, r = coeffs.shape
    return _check(lib().s4r_reconstruct(_ptr(coeffs), n_total, _ptr(basis), basis.shape[0], r,
                                        _ptr(rows), rows.numel(), _ptr(out), _DTYPE[coeffs.dtype],
                                        _stream(stream)), "s4r_reconstruct")


def s4r_read_device_status(workspace, stream=None) -> int:
    """Synchronise the stream and return the sticky device status code."""
    return int(lib().s4r_read_device_status(_ptr(workspace), _stream(stream)))


def s4r_debug_waits(limit_cycles: int = 0, unreachable_barrier: bool = False) -> int:
    """Testing hook: limit of the device-side bounded waits (SM cycles, 0 =
    default) and the switch that makes the scoring kernel's grid barrier
    unreachable (see include/s4r.h)."""
    return _check(lib().s4r_debug_waits(int(limit_cycles), 1 if unreachable_barrier else 0),
                  "s4r_debug_waits")


def s4r_clear_device_status(workspace, stream=None) -> int:
    return _check(lib().s4r_clear_device_status(_ptr(workspace), _stream(stream)),
                  "s4r_clear_device_status")
