"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on
seeded inputs at sizes the oracle finishes in seconds (several blocks, ragged
tails, several scan segments), plus edge cases."""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, assert_close_bf16_out, assert_close_heads,
                             f64, lam)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _reset_tuning():
    L.la_set_tuning(0, 0)
    yield
    L.la_set_tuning(0, 0)


def _prefill(q, k, v, s, out_dtype):
    B, H, N, d = q.shape
    o = torch.full(q.shape, float("nan"), dtype=out_dtype, device=DEV)
    st = torch.full((B, H, d, d), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d, 0, q.dtype)
    L.la_prefill(q, k, v, s, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    return o, st


# ---------------------------------------------------------------- fp32 path

def test_tiny_fp32_config():
    """B=1, H=2, N=256, d=64, fp32, block 64: O [1,2,256,64] and the 64x64 states."""
    q, k, v, s = inputs.prefill_inputs(1, 2, 256, 64, torch.float32, DEV, seed=0)
    L.la_set_tuning(64, 0)
    o, st = _prefill(q, k, v, s, torch.float32)
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o), o_ref, TOL_F32, "O")
    assert_close(f64(st), st_ref, TOL_F32, "state")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [32, 64, 128])
def test_fp32_block_invariance(d, block):
    q, k, v, s = inputs.prefill_inputs(2, 3, 301, d, torch.float32, DEV, seed=1)
    L.la_set_tuning(block, 0)
    o, st = _prefill(q, k, v, s, torch.float32)
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o), o_ref, TOL_F32, f"O C={block}")
    assert_close(f64(st), st_ref, TOL_F32, f"state C={block}")


# ---------------------------------------------------------------- bf16 tensor-core path

@pytest.mark.parametrize("N", [1, 127, 128, 129, 700, 1000])
def test_bf16_prefill_lengths(N):
    q, k, v, s = inputs.prefill_inputs(2, 3, N, 128, torch.bfloat16, DEV, seed=N)
    o, st = _prefill(q, k, v, s, torch.float32)
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o), o_ref, TOL_BF16, "O")
    assert_close(f64(st), st_ref, TOL_BF16, "state")


@pytest.mark.parametrize("seg", [128, 256, 384, 1024])
def test_bf16_segment_scan_invariance(seg):
    """Different scan segmentations give the same result (within tolerance)."""
    q, k, v, s = inputs.prefill_inputs(1, 4, 1500, 128, torch.bfloat16, DEV, seed=7)
    L.la_set_tuning(0, seg)
    o, st = _prefill(q, k, v, s, torch.float32)
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o), o_ref, TOL_BF16, f"O seg={seg}")
    assert_close(f64(st), st_ref, TOL_BF16, f"state seg={seg}")


def test_bf16_output_dtype():
    q, k, v, s = inputs.prefill_inputs(1, 4, 777, 128, torch.bfloat16, DEV, seed=3)
    L.la_set_tuning(0, 256)
    o, _ = _prefill(q, k, v, s, torch.bfloat16)
    o_ref, _ = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close_bf16_out(f64(o), o_ref, TOL_BF16, "bf16 O")


def test_bf16_decay_extremes():
    """lam = 1 (slope 0: plain causal linear attention) and lam ~ 0 (slope 20)."""
    q, k, v, _ = inputs.prefill_inputs(1, 3, 600, 128, torch.bfloat16, DEV, seed=4)
    s = torch.tensor([0.0, 20.0, 0.01], dtype=torch.float32, device=DEV)
    L.la_set_tuning(0, 256)
    o, st = _prefill(q, k, v, s, torch.float32)
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    for h in range(3):
        assert_close(f64(o)[:, h], o_ref[:, h], TOL_BF16, f"O head {h}")
        assert_close(f64(st)[:, h], st_ref[:, h], TOL_BF16, f"state head {h}")


def test_bf16_zero_length():
    q = torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device=DEV)
    s = inputs.slopes(2, DEV)
    st = torch.full((1, 2, 128, 128), float("nan"), device=DEV)
    o = torch.empty_like(q, dtype=torch.float32)
    ws = L.workspace(L.LA_OP_PREFILL, 1, 2, 0, 128, 0, torch.bfloat16)
    L.la_prefill(q, q, q, s, o, st, ws)
    torch.cuda.synchronize()
    assert torch.all(st == 0)


# ---------------------------------------------------------------- varlen

@pytest.mark.parametrize("seg", [0, 256])
def test_varlen(seg):
    lengths = [300, 0, 1, 1029, 128, 2000, 77]
    q, k, v, cu, s = inputs.varlen_inputs(lengths, 4, 128, torch.bfloat16, DEV, seed=5)
    L.la_set_tuning(0, seg)
    S = len(lengths)
    o = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    st = torch.full((S, 4, 128, 128), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, 4, q.shape[1], 128, S, torch.bfloat16)
    L.la_prefill_varlen(cu, q, k, v, s, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    o_ref, st_ref = oracle.forward_varlen(cu.cpu().numpy(), f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o), o_ref, TOL_BF16, "O")
    assert_close(f64(st), st_ref, TOL_BF16, "state")
    assert torch.all(st[1] == 0)


def test_varlen_many_items_longest_first():
    """Enough (sequence, head, half) items that each sequence is one segment and
    the planner orders them by length (empty, one-token, partial and whole
    blocks among them); heads 0 and 63 checked by the quadratic oracle."""
    lengths = [0, 300, 1, 128, 0, 1000, 129, 50, 2048, 7]
    H = 64
    q, k, v, cu, s = inputs.varlen_inputs(lengths, H, 128, torch.bfloat16, DEV, seed=15)
    S = len(lengths)
    o = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    st = torch.full((S, H, 128, 128), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, q.shape[1], 128, S, torch.bfloat16)
    L.la_prefill_varlen(cu, q, k, v, s, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = [0, 63]
    sub = lambda t: np.stack([f64(t[h]) for h in hs])
    o_ref, st_ref = oracle.forward_varlen(cu.cpu().numpy(), sub(q), sub(k), sub(v), lam(s)[hs])
    assert_close(sub(o), o_ref, TOL_BF16, "O (heads 0, 63)")
    assert_close(np.stack([f64(st[:, h]) for h in hs], axis=1), st_ref, TOL_BF16, "states")
    assert torch.all(st[0] == 0) and torch.all(st[4] == 0)
    assert not torch.isnan(o).any()


def test_varlen_matches_separate_calls():
    lengths = [513, 1200, 64]
    q, k, v, cu, s = inputs.varlen_inputs(lengths, 2, 128, torch.bfloat16, DEV, seed=6)
    o, st = L.prefill_varlen(cu, q, k, v, s, out_dtype=torch.float32)
    c = cu.tolist()
    for i in range(len(lengths)):
        sl = slice(c[i], c[i + 1])
        o_i, st_i = L.prefill(q[None, :, sl].contiguous(), k[None, :, sl].contiguous(),
                              v[None, :, sl].contiguous(), s, out_dtype=torch.float32)
        assert_close(f64(o[:, sl]), f64(o_i[0]), TOL_BF16, f"O seq {i}")
        assert_close(f64(st[i]), f64(st_i[0]), TOL_BF16, f"state seq {i}")


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 128)])
def test_decode(dtype, d):
    q, k, v, state, s = inputs.decode_inputs(8, 4, d, dtype, DEV, seed=8)
    st_ref_in = f64(state)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    L.la_decode(q, k, v, s, state, o)
    o_ref, st_ref = oracle.decode(f64(q), f64(k), f64(v), lam(s), st_ref_in)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert_close(f64(o), o_ref, tol, "o")
    assert_close(f64(state), st_ref, tol, "state")


def test_prefill_then_decode_chain():
    """prefill(N - m) state + m decode steps == last m rows / final state of prefill(N)."""
    N, m = 900, 4
    q, k, v, s = inputs.prefill_inputs(1, 4, N, 128, torch.bfloat16, DEV, seed=9)
    o_full, st_full = L.prefill(q, k, v, s, out_dtype=torch.float32)
    _, st = L.prefill(q[:, :, :N - m].contiguous(), k[:, :, :N - m].contiguous(),
                      v[:, :, :N - m].contiguous(), s, out_dtype=torch.float32)
    for t in range(N - m, N):
        o_t = L.decode(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(),
                       s, st, out_dtype=torch.float32)
        assert_close(f64(o_t), f64(o_full[:, :, t]), TOL_BF16, f"row {t}")
    assert_close(f64(st), f64(st_full), TOL_BF16, "state")


# ---------------------------------------------------------------- backward

@pytest.mark.parametrize("seg", [0, 256])
def test_backward(seg):
    q, k, v, s = inputs.prefill_inputs(1, 3, 700, 128, torch.bfloat16, DEV, seed=10)
    do = inputs.grad_output(q.shape, torch.bfloat16, DEV, seed=11)
    L.la_set_tuning(0, seg)
    dq, dk, dv = L.backward(do, q, k, v, s, out_dtype=torch.float32)
    rq, rk, rv = oracle.backward(f64(do), f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(dq), rq, TOL_BF16, "dQ")
    assert_close(f64(dk), rk, TOL_BF16, "dK")
    assert_close(f64(dv), rv, TOL_BF16, "dV")


def test_backward_fp32_path():
    q, k, v, s = inputs.prefill_inputs(1, 2, 200, 64, torch.float32, DEV, seed=12)
    do = inputs.grad_output(q.shape, torch.float32, DEV, seed=13)
    dq, dk, dv = L.backward(do, q, k, v, s)
    rq, rk, rv = oracle.backward(f64(do), f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(dq), rq, TOL_F32, "dQ")
    assert_close(f64(dk), rk, TOL_F32, "dK")
    assert_close(f64(dv), rv, TOL_F32, "dV")


def test_bf16_many_items_per_cta_segmented():
    """Two-block scan segments, ~10 items per CTA: every non-last segment runs a
    phase A whose second decayed-value buffer shares Q slot 0 with phase C."""
    q, k, v, s = inputs.prefill_inputs(2, 64, 1500, 128, torch.bfloat16, DEV, seed=70)
    L.la_set_tuning(0, 256)
    try:
        o, st = _prefill(q, k, v, s, torch.float32)
    finally:
        L.la_set_tuning(0, 0)
    o_ref, st_ref = oracle.recurrence(f64(q), f64(k), f64(v), lam(s))
    assert_close_heads(f64(o), o_ref, TOL_BF16, range(64), "O", axis=1)
    assert_close_heads(f64(st), st_ref, TOL_BF16, range(64), "state", axis=1)
