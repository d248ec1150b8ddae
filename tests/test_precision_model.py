"""The precision design of the tensor-core prefill, checked on CPU.

A model of the kernel's tiled algorithm in fp64 numpy: 128-token blocks,
P = (Q K^T) * lam^(i-j) [j <= i], O = P V + lam^(i+1) Q S, the decayed values
lam^(L-1-j) v_j, S = lam^L S + K^T Vd. The bf16 roundings the kernel applies
to the three operands it forms itself (P, the state copy, the decayed values)
are emulated, either as the kernel does them (x = hi + lo, both bf16) or as a
single bf16 rounding. Compared with the fp64 oracle on the prefill
workload's inputs (eight of the 64 heads' decays, 3000 tokens):

  * in exact arithmetic the tiled model reproduces the oracle, which checks
    the kernel's decay bookkeeping independently of the GPU;
  * with every operand split hi + lo the error is far inside the 1e-2 of rms
    gate;
  * a single bf16 rounding of P, or of the decayed values, misses the gate,
    and one of the state copy reaches it: the reason each is split.
This is a model of the numerics, not of the CUDA path; the GPU parity tests
check the kernels themselves.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_02_b200 import inputs


def _round(x, mode):
    if mode == "exact":
        return x
    bf = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()
    if mode == "bf16":
        return bf
    if mode == "split":
        return bf + _round(x - bf, "bf16")
    raise ValueError(mode)


def _tiled(q, k, v, lam, p_mode, s_mode, v_mode, C=128):
    N, d = q.shape
    O = np.zeros((N, d))
    S = np.zeros((d, d))
    pw = lam ** np.arange(C + 1)
    for t0 in range(0, N, C):
        L = min(C, N - t0)
        Q, K, V = q[t0:t0 + L], k[t0:t0 + L], v[t0:t0 + L]
        i, j = np.arange(L)[:, None], np.arange(L)[None, :]
        P = _round((Q @ K.T) * np.where(j <= i, pw[np.clip(i - j, 0, C)], 0.0), p_mode)
        O[t0:t0 + L] = P @ V + pw[1:L + 1][:, None] * (Q @ _round(S, s_mode))
        Vd = _round(V * pw[L - 1 - np.arange(L)][:, None], v_mode)
        S = pw[L] * S + K.T @ Vd
    return O, S


@pytest.fixture(scope="module")
def case():
    N, H = 3000, 8
    q, k, v, _ = inputs.prefill_inputs(1, H, N, 128, torch.bfloat16, "cpu", seed=N)
    lam = oracle.lambdas_from_slopes(inputs.slopes(64)[::64 // H][:H].numpy())
    f = lambda t: t.to(torch.float64).numpy()[0]
    qn, kn, vn = f(q), f(k), f(v)
    o_ref, s_ref = oracle.recurrence(qn[None], kn[None], vn[None], lam)
    return qn, kn, vn, lam, o_ref[0], s_ref[0]


def _errors(case, modes):
    qn, kn, vn, lam, o_ref, s_ref = case
    res = [_tiled(qn[h], kn[h], vn[h], lam[h], *modes) for h in range(len(lam))]
    O = np.stack([r[0] for r in res])
    S = np.stack([r[1] for r in res])
    rms = lambda x: float(np.sqrt(np.mean(x * x)))
    return (float(np.abs(O - o_ref).max()) / rms(o_ref),
            float(np.abs(S - s_ref).max()) / rms(s_ref))


def test_tiled_model_in_exact_arithmetic_is_the_operator(case):
    eo, es = _errors(case, ("exact", "exact", "exact"))
    assert eo < 1e-12 and es < 1e-12


def test_hi_lo_splits_stay_far_inside_the_gate(case):
    eo, es = _errors(case, ("split", "split", "split"))
    assert eo < 1e-3 and es < 1e-3, (eo, es)      # about 3e-5 of rms


def test_single_bf16_roundings_miss_or_reach_the_gate(case):
    eo_p, _ = _errors(case, ("bf16", "split", "split"))
    eo_s, _ = _errors(case, ("split", "bf16", "split"))
    eo_v, es_v = _errors(case, ("split", "split", "bf16"))
    assert eo_p > 1e-2, eo_p                       # P rounded once: about 1.7e-2
    assert eo_v > 1e-2 and es_v > 1e-2, (eo_v, es_v)  # decayed values: 1.7e-2, state 1.4e-2
    assert eo_s > 0.5e-2, eo_s                     # state copy: about 1.1e-2
