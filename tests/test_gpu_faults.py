"""Failure detection of the chunk-parallel scan, without faulting the GPU.

The only device-side wait on another CTA is a segment waiting for its
predecessor's prefix state. It is bounded: when it runs out, the kernel
records LA_ERR_TIMEOUT in the workspace and finishes, and the host reads the
status. Here the host injects the failure (predecessors never signal) with a
short limit, checks the status, then checks that the context still works.
"""
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import TOL_BF16, assert_close, f64, lam

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_scan_wait_times_out_and_context_survives():
    q, k, v, s = inputs.prefill_inputs(1, 2, 1024, 128, torch.bfloat16, DEV, seed=31)
    o = torch.empty(q.shape, dtype=torch.float32, device=DEV)
    ws = L.workspace(L.LA_OP_PREFILL, 1, 2, 1024, 128)
    try:
        L.la_set_tuning(0, 256)                 # 4 segments per head: 3 waits each
        L.la_set_fault_injection(1, 20000)      # predecessors never signal; 20 ms limit
        L.la_prefill(q, k, v, s, o, None, ws)   # the launch itself succeeds
        assert L.la_read_device_status(ws) == L.LA_ERR_TIMEOUT
    finally:
        L.la_set_fault_injection(0, 0)
    # Same context, normal operation: correct results and a clean status.
    o2, st2 = L.prefill(q, k, v, s, out_dtype=torch.float32)
    ws2 = L.workspace(L.LA_OP_PREFILL, 1, 2, 1024, 128)
    L.la_prefill(q, k, v, s, o2, st2, ws2)
    assert L.la_read_device_status(ws2) == L.LA_OK
    o_ref, _ = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    assert_close(f64(o2), o_ref, TOL_BF16, "O after the injected timeout")
    L.la_set_tuning(0, 0)
