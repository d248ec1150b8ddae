"""Lightning attention fp64 CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The product path (the CUDA library and its Python
binding) never imports it, and it imports nothing from the product path.

It wraps ``lightning_oracle.c`` (plain C, fp64, OpenMP) through ctypes. Every
function takes float64 numpy arrays, which callers build from the exact input
values the GPU sees (bf16 and fp32 both convert to float64 without rounding).

Operator (per (sequence, head) problem, head dim d = d_k = d_v):

    O_i   = sum_{j<=i} lam^(i-j) (q_i . k_j) v_j
    state = sum_j lam^(N-1-j) k_j^T v_j           ([d_k][d_v])

after "MiniMax-01: Scaling Foundation Models with Lightning Attention |
Summary", section 2.2 (Linear Attention); the per-head decay lam = exp(-s) is
this library's stated operator definition (the page's derivation omits it).

Every function here is pinned by tests/test_oracle_pins.py (hand-derived
fixtures, exact rational brute force, closed forms, invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "lightning_oracle.c")
LIBRARY = os.path.join(_HERE, "liblightning_oracle.so")


def build(force: bool = False, src: str = SOURCE, out: str = LIBRARY) -> str:
    """Compile the oracle with gcc (fp64, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
               "-o", out, src, "-lm"]
        subprocess.check_call(cmd)
    return out


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i64(a):
    return np.ascontiguousarray(a, dtype=np.int64)


def _out(shape):
    """Output buffers start as NaN, so any element the C code fails to write shows."""
    return np.full(shape, np.nan)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lambdas_from_slopes(slopes) -> np.ndarray:
    """lam_h = exp(-s_h), evaluated in fp64."""
    return np.exp(-np.asarray(slopes, dtype=np.float64))


def _dense_problems(B, H, N, lam):
    lam = np.asarray(lam, dtype=np.float64).reshape(-1)
    p = np.arange(B * H)
    return _i64(p * N), _i64(np.full(B * H, N)), _i64(p), _f64(np.tile(lam, B))


def _varlen_problems(cu_seqlens, H, T, lam):
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lam = np.asarray(lam, dtype=np.float64).reshape(-1)
    ro, ln, so, lp = [], [], [], []
    for s in range(len(cu) - 1):
        for h in range(H):
            ro.append(h * T + cu[s])
            ln.append(cu[s + 1] - cu[s])
            so.append(s * H + h)
            lp.append(lam[h])
    return _i64(ro), _i64(ln), _i64(so), _f64(lp)


class Oracle:
    """ctypes binding of one build of ``lightning_oracle.c``."""

    def __init__(self, path: str | None = None):
        lib = ctypes.CDLL(path or build())
        P, L, I, D = ctypes.c_void_p, ctypes.c_long, ctypes.c_int, ctypes.c_double
        lib.oracle_forward.argtypes = [I, P, P, P, P, P, P, P, P, P, L]
        lib.oracle_forward_from_state.argtypes = [I, P, P, P, P, P, P, P, P, P, P, L]
        lib.oracle_recurrence.argtypes = [I, P, P, P, P, P, P, P, P, P, P, L, I]
        lib.oracle_backward.argtypes = [I, P, P, P, P, P, P, P, P, P, P, L]
        lib.oracle_decode.argtypes = [P, P, P, P, P, P, L, L]
        lib.oracle_norm_gate.argtypes = [P, P, P, D, P, L, L, L, L]
        lib.oracle_state_prefix.argtypes = [P, P, P, L, L, L, L, P]
        lib.oracle_forward_rows.argtypes = [P, P, P, P, L, P, L, D]
        for f in ("oracle_forward", "oracle_forward_from_state", "oracle_recurrence", "oracle_backward", "oracle_decode",
                  "oracle_forward_rows", "oracle_norm_gate", "oracle_state_prefix"):
            getattr(lib, f).restype = None
        self.lib = lib

    def forward(self, q, k, v, lam, state_in=None):
        """Quadratic form over [B,H,N,d]. Returns (O [B,H,N,d], state [B,H,d,d]).
        state_in [B,H,d,d]: the state of a prefix before token 0 (None = no prefix)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, N, d = q.shape
        ro, ln, so, lp = _dense_problems(B, H, N, lam)
        o = _out(q.shape)
        st = _out((B, H, d, d))
        if state_in is None:
            self.lib.oracle_forward(B * H, _p(ro), _p(ln), _p(so), _p(lp), _p(q), _p(k), _p(v),
                                    _p(o), _p(st), d)
        else:
            si = _f64(state_in).reshape(B, H, d, d)
            self.lib.oracle_forward_from_state(B * H, _p(ro), _p(ln), _p(so), _p(lp), _p(q),
                                               _p(k), _p(v), _p(si), _p(o), _p(st), d)
        return o, st

    def recurrence(self, q, k, v, lam, state_in=None, reverse=False, want_o=True):
        """Token recurrence over [B,H,N,d]. Returns (O or None, final state [B,H,d,d])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, N, d = q.shape
        ro, ln, so, lp = _dense_problems(B, H, N, lam)
        o = _out(q.shape) if want_o else None
        si = None if state_in is None else _f64(state_in)
        st = _out((B, H, d, d))
        self.lib.oracle_recurrence(B * H, _p(ro), _p(ln), _p(so), _p(lp), _p(q), _p(k), _p(v),
                                   _p(o), _p(si), _p(st), d, 1 if reverse else 0)
        return o, st

    def forward_varlen(self, cu_seqlens, q, k, v, lam, state_in=None):
        """Quadratic form per packed sequence, [H,T,d]. Returns (O, state [S,H,d,d]).
        state_in [S,H,d,d]: each sequence's prefix state (None = no prefix)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        H, T, d = q.shape
        ro, ln, so, lp = _varlen_problems(cu_seqlens, H, T, lam)
        o = _out(q.shape)
        st = _out((len(cu_seqlens) - 1, H, d, d))
        if state_in is None:
            self.lib.oracle_forward(len(ro), _p(ro), _p(ln), _p(so), _p(lp), _p(q), _p(k),
                                    _p(v), _p(o), _p(st), d)
        else:
            si = _f64(state_in).reshape(len(cu_seqlens) - 1, H, d, d)
            self.lib.oracle_forward_from_state(len(ro), _p(ro), _p(ln), _p(so), _p(lp), _p(q),
                                               _p(k), _p(v), _p(si), _p(o), _p(st), d)
        return o, st

    def recurrence_varlen(self, cu_seqlens, q, k, v, lam, want_o=True, state_in=None):
        """Token recurrence per packed sequence, [H,T,d]. Returns (O, state [S,H,d,d])."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        H, T, d = q.shape
        ro, ln, so, lp = _varlen_problems(cu_seqlens, H, T, lam)
        o = _out(q.shape) if want_o else None
        st = _out((len(cu_seqlens) - 1, H, d, d))
        si = None if state_in is None else _f64(state_in)
        self.lib.oracle_recurrence(len(ro), _p(ro), _p(ln), _p(so), _p(lp), _p(q), _p(k),
                                   _p(v), _p(o), _p(si), _p(st), d, 0)
        return o, st

    def forward_rows(self, q, k, v, lam, rows):
        """Quadratic form of one head ([N,d]) at the given rows. Returns [len(rows), d]."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        N, d = q.shape
        rows = _i64(rows)
        out = _out((len(rows), d))
        self.lib.oracle_forward_rows(_p(q), _p(k), _p(v), _p(rows), len(rows), _p(out), d,
                                     float(lam))
        return out

    def decode(self, q, k, v, lam, state):
        """One decode step. q,k,v [B,H,d]; state [B,H,d,d] (left untouched).
        Returns (o [B,H,d], updated state)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, d = q.shape
        st = _f64(state).copy()
        lp = _f64(np.tile(np.asarray(lam, dtype=np.float64).reshape(-1), B))
        o = _out((B, H, d))
        self.lib.oracle_decode(_p(q), _p(k), _p(v), _p(lp), _p(st), _p(o), B * H, d)
        return o, st

    def norm_gate(self, o, g, w, eps):
        """RMS normalization over the H*d features of each token, then a sigmoid
        gate. o [B,H,N,d] (head-major); g [B,N,H*d]; w [H*d]. Returns Y [B,N,H*d]."""
        o, g, w = _f64(o), _f64(g), _f64(w)
        B, H, N, d = o.shape
        y = _out((B, N, H * d))
        self.lib.oracle_norm_gate(_p(o), _p(g), _p(w), float(eps), _p(y), B, H, N, d)
        return y

    def state_prefix(self, states, lam, lens, r):
        """Incoming state of chunk r from the local states of consecutive chunks.
        states [R,B,H,d,d] (each chunk's own state); lam [H]; lens [R].
        Returns [B,H,d,d]."""
        states = _f64(states)
        R, B, H, d, _ = states.shape
        lp = _f64(np.tile(np.asarray(lam, dtype=np.float64).reshape(-1), B))
        ln = _i64(lens)
        out = _out((B, H, d, d))
        self.lib.oracle_state_prefix(_p(states), _p(lp), _p(ln), R, int(r), B * H, d, _p(out))
        return out

    def backward(self, dout, q, k, v, lam):
        """Quadratic-sum gradients of <dO, O>, all [B,H,N,d]. Returns (dQ, dK, dV)."""
        dout, q, k, v = _f64(dout), _f64(q), _f64(k), _f64(v)
        B, H, N, d = q.shape
        ro, ln, _, lp = _dense_problems(B, H, N, lam)
        dq, dk, dv = _out(q.shape), _out(q.shape), _out(q.shape)
        self.lib.oracle_backward(B * H, _p(ro), _p(ln), _p(lp), _p(dout), _p(q), _p(k), _p(v),
                                 _p(dq), _p(dk), _p(dv), d)
        return dq, dk, dv

    def backward_recurrence(self, dout, q, k, v, lam):
        """Gradients by three token recurrences (O(N d^2) per head), for large shapes:
        dQ = forward recurrence with (q,k,v) <- (dO, V, K);
        dK = reverse recurrence with (q,k,v) <- (V, dO, Q);
        dV = reverse recurrence with (q,k,v) <- (K, Q, dO)."""
        dq, _ = self.recurrence(dout, v, k, lam)
        dk, _ = self.recurrence(v, dout, q, lam, reverse=True)
        dv, _ = self.recurrence(k, q, dout, lam, reverse=True)
        return dq, dk, dv


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def forward(*a, **kw):
    return default().forward(*a, **kw)


def recurrence(*a, **kw):
    return default().recurrence(*a, **kw)


def forward_varlen(*a, **kw):
    return default().forward_varlen(*a, **kw)


def recurrence_varlen(*a, **kw):
    return default().recurrence_varlen(*a, **kw)


def forward_rows(*a, **kw):
    return default().forward_rows(*a, **kw)


def decode(*a, **kw):
    return default().decode(*a, **kw)


def backward(*a, **kw):
    return default().backward(*a, **kw)


def norm_gate(*a, **kw):
    return default().norm_gate(*a, **kw)


def state_prefix(*a, **kw):
    return default().state_prefix(*a, **kw)


def backward_recurrence(*a, **kw):
    return default().backward_recurrence(*a, **kw)
