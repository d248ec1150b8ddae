"""Helpers shared by the GPU parity tests (comparison against the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances: max |X - X_ref| <= TOL * rms(X_ref) over the compared tensor.
TOL_BF16 = 1e-2   # bf16 inputs, fp32 accumulation, fp32 outputs
TOL_F32 = 1e-4    # fp32 path
BF16_ULP = 2.0 ** -8  # extra elementwise allowance when the output itself is bf16


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def lam(slopes: torch.Tensor) -> np.ndarray:
    return oracle.lambdas_from_slopes(slopes.cpu().numpy())


def rms(x) -> float:
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def err_ratio(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    r = rms(ref)
    if r == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref))) / r


def assert_close(got, ref, tol, what=""):
    e = err_ratio(got, ref)
    assert np.all(np.isfinite(np.asarray(got))), f"{what}: non-finite values"
    assert e <= tol, f"{what}: max|err|/rms = {e:.3e} > {tol:.1e}"
    return e


def assert_close_bf16_out(got, ref, tol, what=""):
    """Elementwise |got - ref| <= tol * rms(ref) + 2^-8 |ref| (bf16-rounded outputs)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = tol * rms(ref) + BF16_ULP * np.abs(ref)
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond tol*rms + 2^-8|ref|"


def assert_close_heads(got, ref, tol, heads, what="", axis=0):
    """The tolerance over the compared tensor, and again inside each head:
    max |err| <= tol * rms(ref of that head), so that a fast-decay head with a
    small output cannot hide its errors under a slow head's larger rms.
    `axis` is the head axis of `got` and `ref`; `heads` names its entries."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    worst = assert_close(got, ref, tol, what)
    for i, h in enumerate(heads):
        e = assert_close(np.take(got, i, axis=axis), np.take(ref, i, axis=axis), tol,
                         f"{what}, head {h} alone")
        worst = max(worst, e)
    return worst
