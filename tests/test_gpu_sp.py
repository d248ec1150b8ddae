"""GPU parity of the sequence-parallel prefill (LASP+) against the fp64 oracle.

One GPU stands in for R ranks in one process: every chunk's local state is
computed first, then each "rank" runs sp.sp_prefill with a gather that returns
the stacked states (what the all-gather returns on R GPUs). No kernel waits on
another rank, so nothing depends on ranks running at the same time. The
all-gather itself is tested across two gloo ranks in test_multirank_cpu.py."""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs, sp
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, assert_close_heads, f64, lam

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("R", [1, 3, 64])
def test_state_prefix_kernel(R):
    B, H, d = 2, 3, 128
    g = torch.Generator(device=DEV)
    g.manual_seed(R)
    states = torch.randn((R, B, H, d, d), generator=g, device=DEV)
    s = inputs.slopes(H, DEV)
    lens = [(37 * p) % 300 for p in range(R)]
    for r in sorted({0, 1, R // 2, R - 1, R}):
        out = torch.full((B, H, d, d), float("nan"), device=DEV)
        L.la_state_prefix(states, s, lens, r, out)
        torch.cuda.synchronize()
        want = oracle.state_prefix(f64(states), lam(s), lens, r)
        if r == 0:
            assert torch.count_nonzero(out) == 0
        else:
            assert_close(f64(out), want, TOL_F32, f"S_in({r}) of {R}")


@pytest.mark.parametrize("dtype,d,tol", [(torch.bfloat16, 128, TOL_BF16),
                                         (torch.float32, 64, TOL_F32)])
def test_sp_prefill_emulated_ranks(dtype, d, tol):
    B, H = 1, 4
    lens = [300, 129, 0, 700, 1]
    N = sum(lens)
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, dtype, DEV, seed=50)
    cuts = np.concatenate([[0], np.cumsum(lens)])
    chunk = lambda x, r: x[:, :, cuts[r]:cuts[r + 1]].contiguous()
    R = len(lens)
    # what the all-gather would return: every rank's local state
    ws = [L.workspace(L.LA_OP_PREFILL, B, H, n, d, 0, dtype) for n in lens]
    states = torch.stack([sp.local_state(chunk(k, r), chunk(v, r), s, ws[r]) for r in range(R)])
    outs, st = [], None
    for r in range(R):
        o = torch.full((B, H, lens[r], d), float("nan"), dtype=torch.float32, device=DEV)
        st = torch.full((B, H, d, d), float("nan"), dtype=torch.float32, device=DEV)

        def gather(s_loc, r=r):
            assert torch.equal(s_loc, states[r])  # the same local state as in the first pass
            return states

        sp.sp_prefill(chunk(q, r), chunk(k, r), chunk(v, r), s, lens, r, o, st, gather, ws[r])
        outs.append(o)
    torch.cuda.synchronize()
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(np.concatenate([f64(o) for o in outs], axis=2), o_ref, tol, "O of all chunks")
    assert_close(f64(st), st_ref, tol, "final state (last rank)")


@pytest.mark.parametrize("seg", [0, 256])
@pytest.mark.parametrize("N", [0, 1, 129, 700, 1500])
def test_prefill_state_only_bf16(N, seg):
    """la_prefill_state: the final state alone, from zero and from an incoming state."""
    B, H, d = 2, 3, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=60 + N)
    s_in = inputs.state_inputs(B, H, d, DEV, seed=61)
    L.la_set_tuning(0, seg)
    try:
        ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
        st0 = torch.full((B, H, d, d), float("nan"), device=DEV)
        L.la_prefill_state(k, v, s, None, st0, ws)
        st1 = s_in.clone()
        L.la_prefill_state(k, v, s, st1, st1, ws)        # advanced in place
        assert L.la_read_device_status(ws) == L.LA_OK
    finally:
        L.la_set_tuning(0, 0)
    _, want0 = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    _, want1 = oracle.forward(f64(q), f64(k), f64(v), lam(s), state_in=f64(s_in))
    if N == 0:
        assert torch.count_nonzero(st0) == 0 and torch.equal(st1, s_in)
        return
    assert_close(f64(st0), want0, TOL_BF16, "state from zero")
    assert_close(f64(st1), want1, TOL_BF16, "state from S_in")


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_state_only_fp32(d):
    B, H, N = 1, 3, 301
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.float32, DEV, seed=62)
    s_in = inputs.state_inputs(B, H, d, DEV, seed=63)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d, 0, torch.float32)
    st = torch.full((B, H, d, d), float("nan"), device=DEV)
    L.la_prefill_state(k, v, s, s_in, st, ws)
    torch.cuda.synchronize()
    _, want = oracle.forward(f64(q), f64(k), f64(v), lam(s), state_in=f64(s_in))
    assert_close(f64(st), want, TOL_F32, "state")


def test_prefill_state_only_many_items_per_cta():
    """384 items of five blocks on 148 SMs: the three-stage ring and the two
    decayed-value buffers carry on across items of odd length."""
    B, H, N, d = 3, 64, 520, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=65)
    s_in = inputs.state_inputs(B, H, d, DEV, seed=66)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
    st = s_in.clone()
    L.la_prefill_state(k, v, s, st, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    _, want = oracle.recurrence(f64(q), f64(k), f64(v), lam(s), state_in=f64(s_in), want_o=False)
    assert_close_heads(f64(st), want, TOL_BF16, range(H), "state", axis=1)


def test_prefill_state_only_minimax_size():
    """The 32K x 64 shape, heads 0 and 63 against the oracle's recurrence."""
    B, H, N, d = 1, 64, 32768, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=64)
    ws = L.workspace(L.LA_OP_PREFILL, B, H, N, d)
    st = torch.empty((B, H, d, d), device=DEV)
    L.la_prefill_state(k, v, s, None, st, ws)
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = [0, 63]
    sub = lambda t: np.stack([f64(t[0, h]) for h in hs])[None]
    _, want = oracle.recurrence(sub(q), sub(k), sub(v), lam(s)[hs], want_o=False)
    assert_close(f64(st)[:, hs], want, TOL_BF16, "state (heads 0, 63)")


def test_sp_prefill_minimax_size_eight_ranks():
    """The 32K x 64 workload cut into 8 chunks of 4096 tokens (the configuration
    bench.py times for one rank), all ranks emulated; heads 0 and 63 against the
    oracle's recurrence over the whole sequence."""
    B, H, N, d, R = 1, 64, 32768, 128, 8
    n = N // R
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=70)
    chunk = lambda x, r: x[:, :, r * n:(r + 1) * n].contiguous()
    ws = L.workspace(L.LA_OP_PREFILL, B, H, n, d)
    states = torch.stack([sp.local_state(chunk(k, r), chunk(v, r), s, ws) for r in range(R)])
    o = torch.empty((B, H, N, d), dtype=torch.float32, device=DEV)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=DEV)
    for r in range(R):
        o_r = torch.empty((B, H, n, d), dtype=torch.float32, device=DEV)
        sp.sp_prefill(chunk(q, r), chunk(k, r), chunk(v, r), s, [n] * R, r, o_r, st,
                      lambda _: states, ws)
        o[:, :, r * n:(r + 1) * n] = o_r
    assert L.la_read_device_status(ws) == L.LA_OK
    hs = [0, 63]
    sub = lambda t: np.stack([f64(t[0, h]) for h in hs])[None]
    o_ref, st_ref = oracle.recurrence(sub(q), sub(k), sub(v), lam(s)[hs])
    assert_close(sub(o), o_ref, TOL_BF16, "O (heads 0, 63)")
    assert_close(f64(st)[:, hs], st_ref, TOL_BF16, "final state (heads 0, 63)")
