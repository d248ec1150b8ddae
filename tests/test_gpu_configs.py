"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times (default tuning), against the fp64 oracle on sampled heads and rows.

Workloads (seeded, synthetic):
  * MiniMax-shaped prefill: B=1, H=64, N=32768, d=128, bf16;
  * varlen batched prefill: 16 sequences, lengths uniform in [1024, 65536];
  * long-context prefill: N = 1,048,576;
  * decode, batch 256, fp32 state [256,64,128,128], and the backward pass on the
    MiniMax prefill shape.
The oracle computes whole heads by its token recurrence (pinned against the
quadratic form) and single rows by the quadratic form itself.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import (TOL_BF16, assert_close, assert_close_bf16_out, assert_close_heads,
                            f64, lam)

pytestmark = pytest.mark.gpu

DEV = "cuda"
SAMPLE_HEADS = [0, 21, 42, 63]
# The backward pass: eight heads across the decay range.
BACKWARD_HEADS = [0, 9, 18, 27, 36, 45, 54, 63]


@pytest.fixture(autouse=True)
def _default_tuning():
    L.la_set_tuning(0, 0)
    yield
    torch.cuda.empty_cache()


def _heads(t, hs):
    return np.stack([f64(t[0, h]) for h in hs])[None]


def test_minimax_prefill_32k():
    B, H, N, d = 1, 64, 32768, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=1000)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    ob = torch.empty_like(q)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
    L.la_prefill(q, k, v, s, o, st, ws)
    L.la_prefill(q, k, v, s, ob, None, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = SAMPLE_HEADS
    o_ref, st_ref = oracle.recurrence(_heads(q, hs), _heads(k, hs), _heads(v, hs), lam(s)[hs])
    assert_close_heads(_heads(o, hs), o_ref, TOL_BF16, hs, "O (sampled heads)", axis=1)
    assert_close_heads(np.stack([f64(st[0, h]) for h in hs])[None], st_ref, TOL_BF16, hs,
                       "state", axis=1)
    assert_close_bf16_out(_heads(ob, hs), o_ref, TOL_BF16, "bf16 O (sampled heads)")
    # Single rows by the quadratic form (segment and block boundaries, the end).
    rows = [0, 127, 128, 2047, 2048, 16383, 16384, N - 1]
    for h in (0, 63):
        want = oracle.forward_rows(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), lam(s)[h], rows)
        got = f64(o[0, h])[rows]
        rms = float(np.sqrt(np.mean(o_ref[0, hs.index(h)] ** 2)))
        assert np.max(np.abs(got - want)) <= TOL_BF16 * rms, f"rows of head {h}"


def test_minimax_prefill_32k_with_state():
    """The 32K prefill continued from an incoming state, in place (the launch
    bench.py times for the cached-prefix leg)."""
    B, H, N, d = 1, 64, 32768, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=1002)
    s_in = inputs.state_inputs(B, H, d, DEV, seed=1003)
    st = s_in.clone()
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
    L.la_prefill_with_state(q, k, v, s, st, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = SAMPLE_HEADS
    o_ref, st_ref = oracle.recurrence(_heads(q, hs), _heads(k, hs), _heads(v, hs), lam(s)[hs],
                                      state_in=f64(s_in)[:, hs])
    assert_close_heads(_heads(o, hs), o_ref, TOL_BF16, hs, "O (sampled heads)", axis=1)
    assert_close_heads(f64(st)[:, hs], st_ref, TOL_BF16, hs, "state (sampled heads)", axis=1)


def test_varlen_16_sequences():
    H, d = 64, 128
    lengths = inputs.varlen_lengths(16, 1024, 65536, seed=0)
    q, k, v, cu, s = inputs.varlen_inputs(lengths, H, d, torch.bfloat16, DEV, seed=1001)
    T = q.shape[1]
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    st = torch.empty((16, H, d, d), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, T, d, 16)
    L.la_prefill_varlen(cu, q, k, v, s, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = SAMPLE_HEADS
    sub = lambda t: np.stack([f64(t[h]) for h in hs])
    cu_h = cu.cpu().numpy()
    o_ref, st_ref = oracle.recurrence_varlen(cu_h, sub(q), sub(k), sub(v), lam(s)[hs])
    assert_close_heads(sub(o), o_ref, TOL_BF16, hs, "O (sampled heads)", axis=0)
    assert_close_heads(np.stack([f64(st[:, h]) for h in hs], axis=1), st_ref, TOL_BF16, hs,
                       "states", axis=1)
    # Single rows by the quadratic form: each sequence's first and last rows and
    # the block boundary after its first 128 tokens, for the fastest and the
    # slowest head.
    for h in (0, 63):
        for sq in range(16):
            a, b = int(cu_h[sq]), int(cu_h[sq + 1])
            rows = sorted({0, 127, 128, b - a - 1})
            want = oracle.forward_rows(f64(q[h, a:b]), f64(k[h, a:b]), f64(v[h, a:b]),
                                       lam(s)[h], rows)
            got = f64(o[h, a:b])[rows]
            r = float(np.sqrt(np.mean(o_ref[hs.index(h), a:b] ** 2)))
            assert np.max(np.abs(got - want)) <= TOL_BF16 * r, f"rows of head {h}, seq {sq}"


def test_long_context_1m():
    """The 1M-token prefill, gated on fp32 O at the stated tolerance on four
    heads across the decay range (whole heads by the oracle's recurrence, and
    single rows by the quadratic form), then the bf16-output launch that
    bench.py times, checked elementwise."""
    B, H, N, d = 1, 64, 1 << 20, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=1002)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)  # 34.4 GB
    L.la_prefill(q, k, v, s, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    lm = lam(s)
    refs = {}
    # Two heads per oracle call bounds the host memory (about 5 GB per head).
    for pair in (SAMPLE_HEADS[:2], SAMPLE_HEADS[2:]):
        o_ref, st_ref = oracle.recurrence(_heads(q, pair), _heads(k, pair), _heads(v, pair),
                                          lm[pair])
        assert_close_heads(_heads(o, pair), o_ref, TOL_BF16, pair, f"O (heads {pair})", axis=1)
        assert_close_heads(np.stack([f64(st[0, h]) for h in pair])[None], st_ref, TOL_BF16,
                           pair, f"state (heads {pair})", axis=1)
        for i, h in enumerate(pair):
            refs[h] = o_ref[0, i]
        del o_ref
    rows = [0, 127, 128, 65535, 65536, N // 2, N - 1]
    for h in (0, 63):
        want = oracle.forward_rows(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), lm[h], rows)
        got = f64(o[0, h])[rows]
        r = float(np.sqrt(np.mean(refs[h] ** 2)))
        assert np.max(np.abs(got - want)) <= TOL_BF16 * r, f"rows of head {h}"
    del o
    torch.cuda.empty_cache()
    ob = torch.empty_like(q)
    L.la_prefill(q, k, v, s, ob, None, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    for h in SAMPLE_HEADS:
        assert_close_bf16_out(f64(ob[0, h]), refs[h], TOL_BF16, f"bf16 O (head {h})")


def test_few_heads_long_scan():
    """Few chains, long sequence: the default tuning cuts each chain into many
    segments, so the chunk-parallel scan carries the state across dozens of
    segments (and the time-reversed scan does for the backward legs)."""
    B, H, N, d = 1, 4, 65536, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=1006)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
    L.la_prefill(q, k, v, s, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = list(range(H))
    o_ref, st_ref = oracle.recurrence(_heads(q, hs), _heads(k, hs), _heads(v, hs), lam(s))
    assert_close(_heads(o, hs), o_ref, TOL_BF16, "O")
    assert_close(f64(st), st_ref, TOL_BF16, "state")
    do = inputs.grad_output(q.shape, torch.bfloat16, DEV, seed=1007)
    dq, dk, dv = L.backward(do, q, k, v, s, out_dtype=torch.float32)
    rq, rk, rv = oracle.backward_recurrence(_heads(do, hs), _heads(q, hs), _heads(k, hs),
                                            _heads(v, hs), lam(s))
    assert_close(_heads(dq, hs), rq, TOL_BF16, "dQ")
    assert_close(_heads(dk, hs), rk, TOL_BF16, "dK")
    assert_close(_heads(dv, hs), rv, TOL_BF16, "dV")


def test_decode_batch_256():
    B, H, d = 256, 64, 128
    q, k, v, state, s = inputs.decode_inputs(B, H, d, torch.bfloat16, DEV, seed=1003)
    st_in = f64(state)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    L.la_decode(q, k, v, s, state, o)
    o_ref, st_ref = oracle.decode(f64(q), f64(k), f64(v), lam(s), st_in)
    assert_close(f64(o), o_ref, TOL_BF16, "o")
    assert_close(f64(state), st_ref, TOL_BF16, "state")


def test_backward_minimax_shape():
    B, H, N, d = 1, 64, 32768, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=1004)
    do = inputs.grad_output(q.shape, torch.bfloat16, DEV, seed=1005)
    dq, dk, dv = L.backward(do, q, k, v, s, out_dtype=torch.float32)
    hs = BACKWARD_HEADS
    rq, rk, rv = oracle.backward_recurrence(_heads(do, hs), _heads(q, hs), _heads(k, hs),
                                            _heads(v, hs), lam(s)[hs])
    assert_close_heads(_heads(dq, hs), rq, TOL_BF16, hs, "dQ", axis=1)
    assert_close_heads(_heads(dk, hs), rk, TOL_BF16, hs, "dK", axis=1)
    assert_close_heads(_heads(dv, hs), rv, TOL_BF16, hs, "dV", axis=1)
