"""la_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Such callers (a C or embedded host program without a device allocator, a
plugin whose host forbids allocations after start-up, a latency-critical loop
that must not call cudaMalloc) cannot pass a workspace, so the library runs
the prefill on a fixed scratch array of its own. These tests call it through
the C ABI and compare it with la_prefill on a caller-owned workspace, twice in
a row (the shared array keeps the previous call's contents, so the second call
checks that everything that must start at zero is cleared). This file is
collected last so that a failure here comes after every other test has run.
"""
import ctypes

import pytest
import torch

from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run_noalloc(q, k, v, s, out_dtype):
    B, H, N, d = q.shape
    o = torch.full(q.shape, float("nan"), dtype=out_dtype, device=DEV)
    st = torch.full((B, H, d, d), float("nan"), dtype=torch.float32, device=DEV)
    L.la_prefill_noalloc(q, k, v, s, o, st)
    torch.cuda.synchronize()
    return o, st


@pytest.mark.parametrize("dtype,shape,tol", [
    (torch.bfloat16, (2, 4, 3000, 128), TOL_BF16),   # tensor-core path, several scan segments
    (torch.float32, (1, 2, 256, 64), TOL_F32),        # fp32 path
])
def test_noalloc_matches_prefill_twice(dtype, shape, tol):
    L.la_set_tuning(0, 0)
    q, k, v, s = inputs.prefill_inputs(*shape, dtype, DEV, seed=21)
    ref_o, ref_st = L.prefill(q, k, v, s, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for call in range(2):
        o, st = _run_noalloc(q, k, v, s, torch.float32)
        assert_close(f64(o), f64(ref_o), tol, f"O, call {call}")
        assert_close(f64(st), f64(ref_st), tol, f"state, call {call}")


def test_noalloc_refuses_requests_beyond_its_scratch():
    # 256 (sequence, head) pairs at d = 128 need 32 MiB of scratch > 16 MiB.
    need = L.la_workspace_bytes(L.LA_OP_PREFILL, 4, 64, 4096, 128)
    assert need > (16 << 20)
    P = ctypes.c_void_p
    x = P(256)  # never dereferenced: the size check comes first
    status = L.lib().la_prefill_noalloc(x, x, x, x, x, None, 4, 64, 4096, 128, L.LA_BF16,
                                        L.LA_BF16, None)
    assert status == L.LA_ERR_WORKSPACE
