"""la_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Such callers (a C or embedded host program without a device allocator, a
plugin whose host forbids allocations after start-up, a latency-critical loop
that must not call cudaMalloc) cannot pass a workspace, so the library runs
the prefill on a fixed scratch array of its own. These tests call it through
the C ABI and compare it with la_prefill on a caller-owned workspace and with
the fp64 oracle, twice in a row (the shared array keeps the previous call's
contents, so the second call checks that everything that must start at zero
is cleared). They also check the size limit at its boundary and that a
device-side error reaches the caller through la_noalloc_device_status. This
file is collected last so that a failure here comes after every other test
has run.
"""
import ctypes

import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, f64, lam

pytestmark = pytest.mark.gpu

DEV = "cuda"
SCRATCH = 16 << 20  # LA_NOALLOC_SCRATCH_BYTES


def _run_noalloc(q, k, v, s, out_dtype):
    B, H, N, d = q.shape
    o = torch.full(q.shape, float("nan"), dtype=out_dtype, device=DEV)
    st = torch.full((B, H, d, d), float("nan"), dtype=torch.float32, device=DEV)
    L.la_prefill_noalloc(q, k, v, s, o, st)
    assert L.la_noalloc_device_status() == L.LA_OK
    return o, st


@pytest.mark.parametrize("dtype,shape,tol", [
    (torch.bfloat16, (2, 4, 3000, 128), TOL_BF16),   # tensor-core path, several scan segments
    (torch.bfloat16, (1, 127, 520, 128), TOL_BF16),  # 127 (sequence, head) pairs: the scratch nearly full
    (torch.float32, (1, 2, 256, 64), TOL_F32),        # fp32 path
])
def test_noalloc_matches_prefill_and_oracle_twice(dtype, shape, tol):
    L.la_set_tuning(0, 0)
    B, H, N, d = shape
    assert L.la_workspace_bytes(L.LA_OP_PREFILL, B, H, N, d, 0, dtype) <= SCRATCH
    q, k, v, s = inputs.prefill_inputs(*shape, dtype, DEV, seed=21)
    ref_o, ref_st = L.prefill(q, k, v, s, out_dtype=torch.float32)
    torch.cuda.synchronize()
    want_o, want_st = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    for call in range(2):
        o, st = _run_noalloc(q, k, v, s, torch.float32)
        assert_close(f64(o), f64(ref_o), tol, f"O against la_prefill, call {call}")
        assert_close(f64(st), f64(ref_st), tol, f"state against la_prefill, call {call}")
        assert_close(f64(o), want_o, tol, f"O against the oracle, call {call}")
        assert_close(f64(st), want_st, tol, f"state against the oracle, call {call}")


def test_noalloc_refuses_requests_beyond_its_scratch():
    P = ctypes.c_void_p
    x = P(256)  # never dereferenced: the size check comes first
    # 128 (sequence, head) pairs at d = 128: the first size past the limit.
    assert L.la_workspace_bytes(L.LA_OP_PREFILL, 1, 128, 520, 128) > SCRATCH
    assert L.la_workspace_bytes(L.LA_OP_PREFILL, 1, 127, 520, 128) <= SCRATCH
    status = L.lib().la_prefill_noalloc(x, x, x, x, x, None, 1, 128, 520, 128, L.LA_BF16,
                                        L.LA_BF16, None)
    assert status == L.LA_ERR_WORKSPACE
    # 256 pairs need 32 MiB.
    status = L.lib().la_prefill_noalloc(x, x, x, x, x, None, 4, 64, 4096, 128, L.LA_BF16,
                                        L.LA_BF16, None)
    assert status == L.LA_ERR_WORKSPACE


def test_noalloc_reports_a_device_side_timeout():
    """A bounded wait of the scan that gives up is visible to the caller, who
    has no workspace of its own to read: la_noalloc_device_status reads the
    status word in the built-in scratch. The failure is injected on the host
    (predecessors never signal, 20 ms limit); no GPU fault is involved."""
    q, k, v, s = inputs.prefill_inputs(1, 2, 1024, 128, torch.bfloat16, DEV, seed=31)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    try:
        L.la_set_tuning(0, 256)                 # 4 segments per head: 3 waits each
        L.la_set_fault_injection(1, 20000)
        L.la_prefill_noalloc(q, k, v, s, o, None)   # the launch itself succeeds
        assert L.la_noalloc_device_status() == L.LA_ERR_TIMEOUT
    finally:
        L.la_set_fault_injection(0, 0)
        L.la_set_tuning(0, 0)
    # The next call clears the word and computes correct results.
    o2, st2 = _run_noalloc(q, k, v, s, torch.float32)
    want_o, want_st = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o2), want_o, TOL_BF16, "O after the injected timeout")
    assert_close(f64(st2), want_st, TOL_BF16, "state after the injected timeout")
