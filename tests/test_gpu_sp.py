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
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, f64, lam

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
    scratch = [torch.empty((B, H, n, d), dtype=torch.float32, device=DEV) for n in lens]
    ws = [L.workspace(L.LA_OP_PREFILL, B, H, n, d, 0, dtype) for n in lens]
    states = torch.stack([sp.local_state(chunk(q, r), chunk(k, r), chunk(v, r), s, scratch[r],
                                         ws[r]) for r in range(R)])
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
