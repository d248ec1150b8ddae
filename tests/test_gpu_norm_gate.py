"""GPU parity of the output normalization and gate (la_output_norm_gate)
against the fp64 oracle: both input and output dtypes, d = 64 and 128, head
counts from 3 to the 16384-feature limit, the prefill followed by the
norm/gate, and sampled tokens at the MiniMax-shaped size."""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import binding as L
from long_context_02_b200 import inputs
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, assert_close_bf16_out, f64, lam

pytestmark = pytest.mark.gpu

DEV = "cuda"
EPS = 1e-5


def _operands(B, H, N, d, o_dtype, y_dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    o = torch.randn((B, H, N, d), generator=g, device=DEV).to(o_dtype)
    gate = (2 * torch.randn((B, N, H * d), generator=g, device=DEV)).to(y_dtype)
    w = 1 + 0.5 * torch.randn((H * d,), generator=g, device=DEV)
    return o, gate, w


def _check(y, ref, y_dtype, what):
    if y_dtype == torch.float32:
        assert_close(f64(y), ref, TOL_F32, what)
    else:
        assert_close_bf16_out(f64(y), ref, TOL_F32, what)


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("H,d", [(3, 64), (4, 128), (24, 128), (64, 128), (96, 128), (128, 128)])
def test_norm_gate(H, d, o_dtype, y_dtype):
    B, N = 2, 37
    o, gate, w = _operands(B, H, N, d, o_dtype, y_dtype, seed=H * d)
    y = torch.full((B, N, H * d), float("nan"), dtype=y_dtype, device=DEV)
    L.la_output_norm_gate(o, gate, w, EPS, y)
    torch.cuda.synchronize()
    ref = oracle.norm_gate(f64(o), f64(gate), f64(w), EPS)
    _check(y, ref, y_dtype, f"Y H={H} d={d}")


def test_norm_gate_extreme_gates():
    """Saturated and infinite gate inputs give gates of (about) 0 and 1; a NaN
    gate input gives NaN in its own element and leaves the others alone."""
    B, H, N, d = 1, 2, 3, 64
    o, gate, w = _operands(B, H, N, d, torch.float32, torch.float32, seed=7)
    gate[0, 0, :8] = torch.tensor([-1e4, 1e4, float("-inf"), float("inf"), -100.0, 100.0, 0.0,
                                   float("nan")], device=DEV)
    y = torch.empty((B, N, H * d), device=DEV)
    L.la_output_norm_gate(o, gate, w, EPS, y)
    torch.cuda.synchronize()
    ref = oracle.norm_gate(f64(o), f64(gate), f64(w), EPS)
    got = f64(y)
    assert np.isnan(got[0, 0, 7]) and not np.isnan(got[0, 0, :7]).any()
    assert abs(got[0, 0, 0]) < 1e-15 and abs(got[0, 0, 2]) < 1e-15
    np.testing.assert_allclose(got[0, 0, :7], ref[0, 0, :7], rtol=1e-5, atol=1e-15)
    assert_close(got[:, 1:], ref[:, 1:], TOL_F32, "Y (other tokens)")


def test_norm_gate_zero_tokens():
    o = torch.empty((1, 4, 0, 128), dtype=torch.bfloat16, device=DEV)
    g = torch.empty((1, 0, 512), dtype=torch.bfloat16, device=DEV)
    w = torch.ones(512, device=DEV)
    L.la_output_norm_gate(o, g, w, EPS, torch.empty_like(g))
    torch.cuda.synchronize()


def test_prefill_then_norm_gate():
    """The operator's output (fp32, from bf16 inputs) through the norm and gate,
    against the oracle applied to the oracle's own O."""
    B, H, N, d = 1, 4, 700, 128
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, DEV, seed=40)
    o, _ = L.prefill(q, k, v, s, out_dtype=torch.float32, want_state=False)
    _, gate, w = _operands(B, H, N, d, torch.bfloat16, torch.bfloat16, seed=41)
    y = torch.empty((B, N, H * d), dtype=torch.float32, device=DEV)
    L.la_output_norm_gate(o, gate.float(), w, EPS, y)
    torch.cuda.synchronize()
    o_ref, _ = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    ref = oracle.norm_gate(o_ref, f64(gate), f64(w), EPS)
    assert_close(f64(y), ref, TOL_BF16, "Y from the prefill")


def test_norm_gate_minimax_size_sampled_tokens():
    """B=1, H=64, N=32768, d=128 bf16 (the launch bench.py times); tokens
    sampled across the sequence, each against the oracle on the same O."""
    B, H, N, d = 1, 64, 32768, 128
    o, gate, w = _operands(B, H, N, d, torch.bfloat16, torch.bfloat16, seed=42)
    y = torch.empty((B, N, H * d), dtype=torch.bfloat16, device=DEV)
    L.la_output_norm_gate(o, gate, w, EPS, y)
    torch.cuda.synchronize()
    rows = torch.tensor([0, 1, 255, 4096, 16383, 16384, 30001, N - 1], device=DEV)
    ref = oracle.norm_gate(f64(o[:, :, rows]), f64(gate[:, rows]), f64(w), EPS)
    assert_close_bf16_out(f64(y[:, rows]), ref, TOL_F32, "Y (sampled tokens)")
    assert torch.isfinite(y.float()).all()
