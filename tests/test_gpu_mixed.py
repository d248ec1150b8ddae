"""GPU parity of the separated prefill / decode step over a batch of cached
inputs of mixed lengths (la_mixed_step) against the fp64 oracle: one-token
sequences through the decode kernel, longer ones through the prefill from
their states, on two streams or one."""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import (TOL_BF16, TOL_F32, assert_close, assert_close_bf16_out, f64, lam)

pytestmark = pytest.mark.gpu

DEV = "cuda"
# A batch of 20 cached inputs: mostly single tokens, two of 50 tokens (the
# shape of the pages' example), plus an empty input and a multi-block one.
LENGTHS = [1, 1, 50, 1, 1, 1, 0, 1, 1, 1, 1, 1, 300, 1, 1, 50, 1, 1, 1, 1]


@pytest.fixture(autouse=True)
def _reset_tuning():
    L.la_set_tuning(0, 0)
    yield
    L.la_set_tuning(0, 0)


def _mixed(q, k, v, cu, s, s_in, out_dtype, two_streams):
    H, T, d = q.shape
    S = cu.numel() - 1
    o = torch.full(q.shape, float("nan"), dtype=out_dtype, device=DEV)
    st = s_in.clone()
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, T, d, S, q.dtype)
    main = torch.cuda.current_stream()
    if two_streams:
        ps, ds = torch.cuda.Stream(), torch.cuda.Stream()
        ps.wait_stream(main)
        ds.wait_stream(main)
    else:
        ps = ds = main
    L.la_mixed_step(cu, q, k, v, s, st, o, ws, ps, ds)
    main.wait_stream(ps)
    main.wait_stream(ds)
    assert L.la_read_device_status(ws, ps) == L.LA_OK
    torch.cuda.synchronize()
    return o, st


@pytest.mark.parametrize("two_streams", [True, False])
@pytest.mark.parametrize("dtype,d,tol", [(torch.bfloat16, 128, TOL_BF16),
                                         (torch.float32, 64, TOL_F32)])
def test_mixed_step(dtype, d, tol, two_streams):
    H = 4
    q, k, v, cu, s = inputs.varlen_inputs(LENGTHS, H, d, dtype, DEV, seed=30)
    s_in = inputs.state_inputs(len(LENGTHS), H, d, DEV, seed=31)
    o, st = _mixed(q, k, v, cu, s, s_in, torch.float32, two_streams)
    o_ref, st_ref = oracle.forward_varlen(cu.cpu().numpy(), f64(q), f64(k), f64(v), lam(s),
                                          state_in=f64(s_in))
    assert_close(f64(o), o_ref, tol, "O")
    assert_close(f64(st), st_ref, tol, "states")
    assert torch.equal(st[6], s_in[6]), "the empty input keeps its state"
    # the one-token rows alone (decode kernel), against the tolerance of their own rms
    cuh = cu.cpu().numpy()
    one = [int(cuh[i]) for i, n in enumerate(LENGTHS) if n == 1]
    assert_close(f64(o)[:, one], o_ref[:, one], tol, "O of the one-token inputs")


def test_mixed_step_bf16_output_many_heads():
    H, d = 64, 128
    q, k, v, cu, s = inputs.varlen_inputs(LENGTHS, H, d, torch.bfloat16, DEV, seed=32)
    s_in = inputs.state_inputs(len(LENGTHS), H, d, DEV, seed=33)
    o, st = _mixed(q, k, v, cu, s, s_in, torch.bfloat16, True)
    hs = [0, 31, 63]
    sub = lambda t: np.stack([f64(t[h]) for h in hs])
    o_ref, st_ref = oracle.forward_varlen(cu.cpu().numpy(), sub(q), sub(k), sub(v), lam(s)[hs],
                                          state_in=f64(s_in)[:, hs])
    assert_close_bf16_out(sub(o), o_ref, TOL_BF16, "bf16 O (heads 0, 31, 63)")
    assert_close(f64(st)[:, hs], st_ref, TOL_BF16, "states (heads 0, 31, 63)")


@pytest.mark.parametrize("lengths", [[1] * 9, [0, 1, 1, 0], [2, 130, 7, 0], [300]],
                         ids=["all_one_token", "one_token_and_empty", "no_one_token",
                              "single_long"])
def test_mixed_step_edge_batches(lengths):
    """A batch where one of the two parts has nothing to do (or both)."""
    H, d = 4, 128
    q, k, v, cu, s = inputs.varlen_inputs(lengths, H, d, torch.bfloat16, DEV, seed=34)
    s_in = inputs.state_inputs(len(lengths), H, d, DEV, seed=35)
    o, st = _mixed(q, k, v, cu, s, s_in, torch.float32, True)
    o_ref, st_ref = oracle.forward_varlen(cu.cpu().numpy(), f64(q), f64(k), f64(v), lam(s),
                                          state_in=f64(s_in))
    if q.shape[1] > 0:
        assert_close(f64(o), o_ref, TOL_BF16, "O")
    assert_close(f64(st), st_ref, TOL_BF16, "states")


def test_mixed_step_empty_batch():
    H, d = 4, 128
    cu = torch.zeros(1, dtype=torch.int32, device=DEV)
    e = torch.empty((H, 0, d), dtype=torch.bfloat16, device=DEV)
    st = torch.empty((0, H, d, d), device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, 0, d, 0)
    L.la_mixed_step(cu, e, e, e, inputs.slopes(H, DEV), st, e, ws)
    torch.cuda.synchronize()
