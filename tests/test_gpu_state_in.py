"""GPU parity of the prefill continued from an incoming state
(la_prefill_with_state, la_prefill_varlen_with_state) against the fp64 oracle:
both kernels (bf16 tensor-core path and fp32 path), ragged blocks, several scan
segments, the state advanced in place, a prefill cut into pieces, varlen with
empty sequences, and zero length."""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, assert_close_bf16_out, f64, lam)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _reset_tuning():
    L.la_set_tuning(0, 0)
    yield
    L.la_set_tuning(0, 0)


def _run(q, k, v, s, s_in, out_dtype, in_place=False):
    B, H, N, d = q.shape
    o = torch.full(q.shape, float("nan"), dtype=out_dtype, device=DEV)
    if in_place:
        st = s_in.clone()
        src = st
    else:
        st = torch.full((B, H, d, d), float("nan"), dtype=torch.float32, device=DEV)
        src = s_in
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d, 0, q.dtype)
    L.la_prefill_with_state(q, k, v, s, src, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    return o, st


def _ref(q, k, v, s, s_in):
    return oracle.forward(f64(q), f64(k), f64(v), lam(s), state_in=f64(s_in))


@pytest.mark.parametrize("seg", [0, 256])
@pytest.mark.parametrize("N", [1, 129, 700])
def test_bf16_state_in(N, seg):
    q, k, v, s = inputs.prefill_inputs(2, 3, N, 128, torch.bfloat16, DEV, seed=100 + N)
    s_in = inputs.state_inputs(2, 3, 128, DEV, seed=N)
    L.la_set_tuning(0, seg)
    o, st = _run(q, k, v, s, s_in, torch.float32)
    o_ref, st_ref = _ref(q, k, v, s, s_in)
    assert_close(f64(o), o_ref, TOL_BF16, f"O N={N} seg={seg}")
    assert_close(f64(st), st_ref, TOL_BF16, f"state N={N} seg={seg}")


def test_bf16_state_in_in_place_across_segments():
    """state_in and state_out the same array, three scan segments."""
    q, k, v, s = inputs.prefill_inputs(1, 4, 1500, 128, torch.bfloat16, DEV, seed=11)
    s_in = inputs.state_inputs(1, 4, 128, DEV, seed=12)
    L.la_set_tuning(0, 512)
    o, st = _run(q, k, v, s, s_in, torch.float32, in_place=True)
    o_ref, st_ref = _ref(q, k, v, s, s_in)
    assert_close(f64(o), o_ref, TOL_BF16, "O")
    assert_close(f64(st), st_ref, TOL_BF16, "state")


def test_bf16_state_in_bf16_output():
    q, k, v, s = inputs.prefill_inputs(1, 3, 1000, 128, torch.bfloat16, DEV, seed=13)
    s_in = inputs.state_inputs(1, 3, 128, DEV, seed=14)
    o, st = _run(q, k, v, s, s_in, torch.bfloat16)
    o_ref, st_ref = _ref(q, k, v, s, s_in)
    assert_close_bf16_out(f64(o), o_ref, TOL_BF16, "bf16 O")
    assert_close(f64(st), st_ref, TOL_BF16, "state")


@pytest.mark.parametrize("dtype,d,tol", [(torch.bfloat16, 128, TOL_BF16),
                                         (torch.float32, 64, TOL_F32)])
def test_prefill_cut_into_pieces(dtype, d, tol):
    """A prefill cut at arbitrary points (not block multiples), each piece
    continued from the state the previous piece left in place, gives the rows and
    the final state of one prefill over the whole sequence."""
    N = 2000
    q, k, v, s = inputs.prefill_inputs(1, 3, N, d, dtype, DEV, seed=15)
    cuts = [0, 300, 1100, N]
    st = torch.zeros((1, 3, d, d), dtype=torch.float32, device=DEV)
    pieces = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        qa, ka, va = (x[:, :, a:b].contiguous() for x in (q, k, v))
        o = torch.full(qa.shape, float("nan"), dtype=torch.float32, device=DEV)
        ws = L.workspace(L.LA_OP_PREFILL, 1, 3, b - a, d, 0, dtype)
        L.la_prefill_with_state(qa, ka, va, s, st, o, st, ws)
        assert L.la_read_device_status(ws) == L.LA_OK
        pieces.append(f64(o))
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(np.concatenate(pieces, axis=2), o_ref, tol, "O of the pieces")
    assert_close(f64(st), st_ref, tol, "final state")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [32, 128])
def test_fp32_state_in(d, block):
    q, k, v, s = inputs.prefill_inputs(2, 3, 301, d, torch.float32, DEV, seed=16)
    s_in = inputs.state_inputs(2, 3, d, DEV, seed=17)
    L.la_set_tuning(block, 0)
    o, st = _run(q, k, v, s, s_in, torch.float32)
    o_ref, st_ref = _ref(q, k, v, s, s_in)
    assert_close(f64(o), o_ref, TOL_F32, f"O C={block}")
    assert_close(f64(st), st_ref, TOL_F32, f"state C={block}")


def test_zero_length_returns_state_in():
    d = 128
    s = inputs.slopes(4, DEV)
    s_in = inputs.state_inputs(2, 4, d, DEV, seed=18)
    e = torch.empty((2, 4, 0, d), dtype=torch.bfloat16, device=DEV)
    st = torch.full((2, 4, d, d), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, 2, 4, 0, d)
    L.la_prefill_with_state(e, e, e, s, s_in, e, st, ws)
    assert torch.equal(st, s_in)
    st2 = s_in.clone()
    L.la_prefill_with_state(e, e, e, s, st2, e, st2, ws)
    assert torch.equal(st2, s_in)


@pytest.mark.parametrize("dtype,d,seg", [(torch.bfloat16, 128, 0), (torch.bfloat16, 128, 256),
                                         (torch.float32, 64, 0)])
def test_varlen_state_in(dtype, d, seg):
    lengths = [300, 0, 1, 1000, 129]
    H = 4
    q, k, v, cu, s = inputs.varlen_inputs(lengths, H, d, dtype, DEV, seed=19)
    S, T = len(lengths), q.shape[1]
    s_in = inputs.state_inputs(S, H, d, DEV, seed=20)
    L.la_set_tuning(0, seg)
    o = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    st = torch.full((S, H, d, d), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, T, d, S, dtype)
    L.la_prefill_varlen_with_state(cu, q, k, v, s, s_in, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    o_ref, st_ref = oracle.forward_varlen(cu.cpu().numpy(), f64(q), f64(k), f64(v), lam(s),
                                          state_in=f64(s_in))
    tol = TOL_BF16 if dtype == torch.bfloat16 else TOL_F32
    assert_close(f64(o), o_ref, tol, "O")
    assert_close(f64(st), st_ref, tol, "states")
    assert torch.equal(st[1], s_in[1]), "empty sequence keeps its incoming state"


def test_varlen_state_in_many_items_in_place():
    """Enough (sequence, head) items for the longest-first plan; states advanced
    in place; heads 0 and 63 against the oracle's recurrence."""
    lengths = [0, 300, 1, 128, 0, 1000, 129, 50, 2048, 7]
    H, d = 64, 128
    q, k, v, cu, s = inputs.varlen_inputs(lengths, H, d, torch.bfloat16, DEV, seed=21)
    S, T = len(lengths), q.shape[1]
    s_in = inputs.state_inputs(S, H, d, DEV, seed=22)
    st = s_in.clone()
    o = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, T, d, S)
    L.la_prefill_varlen_with_state(cu, q, k, v, s, st, o, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = [0, 63]
    sub = lambda t: np.stack([f64(t[h]) for h in hs])
    o_ref, st_ref = oracle.recurrence_varlen(cu.cpu().numpy(), sub(q), sub(k), sub(v),
                                             lam(s)[hs], state_in=f64(s_in)[:, hs])
    assert_close(sub(o), o_ref, TOL_BF16, "O (heads 0, 63)")
    assert_close(f64(st)[:, hs], st_ref, TOL_BF16, "states (heads 0, 63)")
