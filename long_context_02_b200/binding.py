"""Thin ctypes binding of liblightning.so (argument marshalling only).

Each ``la_*`` function mirrors the C entry point of the same name in
include/lightning.h: it takes torch tensors that already live on the GPU,
derives the sizes from their shapes, passes raw device pointers and the
current CUDA stream, and raises ``LightningError`` on a non-zero status.
Every step of the computation runs in the library's CUDA kernels; there is no
other implementation to fall back to. If the library has not been built,
``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblightning.so")

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT, LA_ERR_WORKSPACE = (
    0, -1, -2, -3, -4, -5)
LA_BF16, LA_F32 = 0, 1
LA_OP_PREFILL, LA_OP_PREFILL_VARLEN, LA_OP_DECODE, LA_OP_BACKWARD = 0, 1, 2, 3

EXPORTED = ["la_workspace_bytes", "la_prefill", "la_prefill_varlen", "la_decode", "la_backward",
            "la_status_string", "la_read_device_status", "la_set_tuning", "la_get_tuning",
            "la_last_launch_count", "la_prefill_noalloc", "la_set_fault_injection",
            "la_prefill_with_state", "la_prefill_varlen_with_state", "la_mixed_step",
            "la_output_norm_gate", "la_state_prefix", "la_prefill_state", "la_noalloc_device_status"]

_lib = None


class LightningError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = lib().la_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} ({status})")


def lib():
    """Load liblightning.so (built in-tree by long_context_02_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m long_context_02_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
        L.la_workspace_bytes.argtypes = [I, I, I, LL, I, I, I]
        L.la_workspace_bytes.restype = SZ
        L.la_prefill.argtypes = [P, P, P, P, P, P, I, I, LL, I, I, I, P, SZ, P]
        L.la_prefill_varlen.argtypes = [P, I, P, P, P, P, P, P, I, LL, I, I, I, P, SZ, P]
        L.la_prefill_with_state.argtypes = [P, P, P, P, P, P, P, I, I, LL, I, I, I, P, SZ, P]
        L.la_prefill_varlen_with_state.argtypes = [P, I, P, P, P, P, P, P, P, I, LL, I, I, I, P,
                                                   SZ, P]
        L.la_mixed_step.argtypes = [P, I, P, P, P, P, P, P, I, LL, I, I, I, P, SZ, P, P]
        L.la_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
        L.la_prefill_state.argtypes = [P, P, P, P, P, I, I, LL, I, I, P, SZ, P]
        L.la_state_prefix.argtypes = [P, P, ctypes.POINTER(LL), I, I, I, I, I, P, P]
        L.la_output_norm_gate.argtypes = [P, P, P, ctypes.c_float, P, I, I, LL, I, I, I, P]
        L.la_backward.argtypes = [P, P, P, P, P, P, P, P, I, I, LL, I, I, I, P, SZ, P]
        L.la_status_string.argtypes = [I]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_read_device_status.argtypes = [P, P]
        L.la_set_tuning.argtypes = [I, I]
        L.la_get_tuning.argtypes = [ctypes.POINTER(I), ctypes.POINTER(I)]
        L.la_last_launch_count.argtypes = []
        L.la_prefill_noalloc.argtypes = [P, P, P, P, P, P, I, I, LL, I, I, I, P]
        L.la_set_fault_injection.argtypes = [I, I]
        L.la_noalloc_device_status.argtypes = [P]
        for f in ("la_prefill", "la_prefill_varlen", "la_prefill_with_state",
                  "la_prefill_varlen_with_state", "la_mixed_step", "la_output_norm_gate",
                  "la_state_prefix", "la_prefill_state",
                  "la_decode", "la_backward",
                  "la_read_device_status", "la_set_tuning", "la_get_tuning",
                  "la_last_launch_count", "la_prefill_noalloc", "la_set_fault_injection",
                  "la_noalloc_device_status"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LA_BF16
    if t.dtype == torch.float32:
        return LA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None or t.numel() == 0:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, status):
    if status != LA_OK:
        raise LightningError(fn, status)


def la_workspace_bytes(op, B, H, N_or_total, d, num_seqs=0, in_dtype=torch.bfloat16) -> int:
    in_t = LA_BF16 if in_dtype == torch.bfloat16 else LA_F32
    return int(lib().la_workspace_bytes(op, B, H, N_or_total, d, num_seqs, in_t))


def workspace(op, B, H, N_or_total, d, num_seqs=0, in_dtype=torch.bfloat16, device="cuda"):
    n = la_workspace_bytes(op, B, H, N_or_total, d, num_seqs, in_dtype)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def la_prefill(q, k, v, slopes, o, state_out, ws, stream=None):
    B, H, N, d = q.shape
    _check("la_prefill", lib().la_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(o), _ptr(state_out), B, H, N, d,
        _dt(q), _dt(o), _ptr(ws), ws.numel(), _stream(stream)))


def la_prefill_varlen(cu_seqlens, q, k, v, slopes, o, state_out, ws, stream=None):
    H, T, d = q.shape
    num_seqs = cu_seqlens.numel() - 1
    _check("la_prefill_varlen", lib().la_prefill_varlen(
        _ptr(cu_seqlens), num_seqs, _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(o),
        _ptr(state_out), H, T, d, _dt(q), _dt(o), _ptr(ws), ws.numel(), _stream(stream)))


def la_prefill_with_state(q, k, v, slopes, state_in, o, state_out, ws, stream=None):
    B, H, N, d = q.shape
    _check("la_prefill_with_state", lib().la_prefill_with_state(
        _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(state_in), _ptr(o), _ptr(state_out),
        B, H, N, d, _dt(q), _dt(o), _ptr(ws), ws.numel(), _stream(stream)))


def la_prefill_varlen_with_state(cu_seqlens, q, k, v, slopes, state_in, o, state_out, ws,
                                 stream=None):
    H, T, d = q.shape
    num_seqs = cu_seqlens.numel() - 1
    _check("la_prefill_varlen_with_state", lib().la_prefill_varlen_with_state(
        _ptr(cu_seqlens), num_seqs, _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(state_in),
        _ptr(o), _ptr(state_out), H, T, d, _dt(q), _dt(o), _ptr(ws), ws.numel(),
        _stream(stream)))


def la_mixed_step(cu_seqlens, q, k, v, slopes, states, o, ws, prefill_stream=None,
                  decode_stream=None):
    H, T, d = q.shape
    num_seqs = cu_seqlens.numel() - 1
    _check("la_mixed_step", lib().la_mixed_step(
        _ptr(cu_seqlens), num_seqs, _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(states),
        _ptr(o), H, T, d, _dt(q), _dt(o), _ptr(ws), ws.numel(), _stream(prefill_stream),
        _stream(decode_stream)))


def la_output_norm_gate(o, gate, weight, eps, y, stream=None):
    B, H, N, d = o.shape
    _check("la_output_norm_gate", lib().la_output_norm_gate(
        _ptr(o), _ptr(gate), _ptr(weight), float(eps), _ptr(y), B, H, N, d, _dt(o), _dt(y),
        _stream(stream)))


def la_state_prefix(states, slopes, lens, r, out, stream=None):
    R, B, H, d, _ = states.shape
    arr = (ctypes.c_longlong * R)(*[int(x) for x in lens])
    _check("la_state_prefix", lib().la_state_prefix(
        _ptr(states), _ptr(slopes), arr, R, int(r), B, H, d, _ptr(out), _stream(stream)))


def la_prefill_state(k, v, slopes, state_in, state_out, ws, stream=None):
    B, H, N, d = k.shape
    _check("la_prefill_state", lib().la_prefill_state(
        _ptr(k), _ptr(v), _ptr(slopes), _ptr(state_in), _ptr(state_out), B, H, N, d, _dt(k),
        _ptr(ws), ws.numel(), _stream(stream)))


def la_decode(q, k, v, slopes, state, o, stream=None):
    B, H, d = q.shape
    _check("la_decode", lib().la_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(state), _ptr(o), B, H, d, _dt(q), _dt(o),
        _stream(stream)))


def la_backward(dout, q, k, v, slopes, dq, dk, dv, ws, stream=None):
    B, H, N, d = q.shape
    _check("la_backward", lib().la_backward(
        _ptr(dout), _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(dq), _ptr(dk), _ptr(dv),
        B, H, N, d, _dt(q), _dt(dq), _ptr(ws), ws.numel(), _stream(stream)))


def la_prefill_noalloc(q, k, v, slopes, o, state_out, stream=None):
    """la_prefill on the library's built-in scratch (for callers that cannot
    allocate device memory; see include/lightning.h)."""
    B, H, N, d = q.shape
    _check("la_prefill_noalloc", lib().la_prefill_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), _ptr(o), _ptr(state_out), B, H, N, d,
        _dt(q), _dt(o), _stream(stream)))


def la_noalloc_device_status(stream=None) -> int:
    """Device-side status of the last la_prefill_noalloc on the current device."""
    return int(lib().la_noalloc_device_status(_stream(stream)))


def la_read_device_status(ws, stream=None) -> int:
    return int(lib().la_read_device_status(_ptr(ws), _stream(stream)))


def la_set_tuning(block_tokens=0, segment_tokens=0):
    _check("la_set_tuning", lib().la_set_tuning(block_tokens, segment_tokens))


def la_get_tuning():
    b, s = ctypes.c_int(), ctypes.c_int()
    lib().la_get_tuning(ctypes.byref(b), ctypes.byref(s))
    return b.value, s.value


def la_set_fault_injection(skip_publish=0, wait_limit_us=0):
    """Test-only: make the scan's inter-segment waits run out (see lightning.h)."""
    _check("la_set_fault_injection", lib().la_set_fault_injection(int(skip_publish),
                                                                 int(wait_limit_us)))


def la_last_launch_count() -> int:
    return int(lib().la_last_launch_count())


def la_status_string(status) -> str:
    return lib().la_status_string(status).decode()


# ---------------------------------------------------------------- conveniences

def prefill(q, k, v, slopes, out_dtype=None, want_state=True, stream=None, state_in=None):
    """Allocate outputs and workspace, run la_prefill (la_prefill_with_state when
    state_in [B,H,d,d] is given). Returns (O, state or None)."""
    B, H, N, d = q.shape
    o = torch.empty_like(q, dtype=out_dtype or q.dtype)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device) if want_state else None
    ws = workspace(LA_OP_PREFILL, B, H, N, d, 0, q.dtype, q.device)
    if state_in is None:
        la_prefill(q, k, v, slopes, o, st, ws, stream)
    else:
        la_prefill_with_state(q, k, v, slopes, state_in, o, st, ws, stream)
    return o, st


def prefill_varlen(cu_seqlens, q, k, v, slopes, out_dtype=None, want_state=True, stream=None,
                   state_in=None):
    H, T, d = q.shape
    S = cu_seqlens.numel() - 1
    o = torch.empty_like(q, dtype=out_dtype or q.dtype)
    st = torch.empty((S, H, d, d), dtype=torch.float32, device=q.device) if want_state else None
    ws = workspace(LA_OP_PREFILL_VARLEN, 1, H, T, d, S, q.dtype, q.device)
    if state_in is None:
        la_prefill_varlen(cu_seqlens, q, k, v, slopes, o, st, ws, stream)
    else:
        la_prefill_varlen_with_state(cu_seqlens, q, k, v, slopes, state_in, o, st, ws, stream)
    return o, st


def decode(q, k, v, slopes, state, out_dtype=None, stream=None):
    o = torch.empty_like(q, dtype=out_dtype or q.dtype)
    la_decode(q, k, v, slopes, state, o, stream)
    return o


def backward(dout, q, k, v, slopes, out_dtype=None, stream=None):
    B, H, N, d = q.shape
    dt = out_dtype or q.dtype
    dq, dk, dv = (torch.empty_like(q, dtype=dt) for _ in range(3))
    ws = workspace(LA_OP_BACKWARD, B, H, N, d, 0, q.dtype, q.device)
    la_backward(dout, q, k, v, slopes, dq, dk, dv, ws, stream)
    return dq, dk, dv
