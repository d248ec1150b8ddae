"""Seeded synthetic inputs shared by the GPU path and the oracle.

This module holds no arithmetic of the method itself: it only draws inputs.
Distributions follow the workloads the library is measured on:

* tiny fp32 case: Q, K, V ~ N(0,1)/sqrt(d);
* MiniMax-shaped bf16 cases (64 heads, head dim 128, as in the MiniMax-01
  README, section 2 "Model Architecture"): Q, K = SiLU(z)/sqrt(d) with
  z ~ N(0,1); V ~ N(0,1); dO ~ N(0,1); rounded to bf16 after the draw;
* decode state ~ N(0, sigma=0.01) in fp32;
* per-head slopes s_h = 2^(-8(h+1)/H), h = 0..H-1 (the decay is lam_h = exp(-s_h)).

Tensors are drawn head by head (so huge tensors never need an fp32 copy of the
whole thing) from one ``torch.Generator`` seeded once, on the requested device.
Callers hand the oracle exact host copies of whatever the GPU received.
"""
from __future__ import annotations

import math

import torch


def slopes(H: int, device="cpu") -> torch.Tensor:
    """s_h = 2^(-8(h+1)/H) as fp32 [H]."""
    s = [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]
    return torch.tensor(s, dtype=torch.float32, device=device)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draw(shape_per_head, H, lead, g, device, dtype, kind, d):
    """Draw a [lead, H, *shape_per_head] tensor head by head."""
    out = torch.empty((lead, H) + tuple(shape_per_head), dtype=dtype, device=device)
    for b in range(lead):
        for h in range(H):
            z = torch.randn(tuple(shape_per_head), generator=g, device=device,
                            dtype=torch.float32)
            if kind == "silu":
                z = torch.nn.functional.silu(z) / math.sqrt(d)
            elif kind == "scaled":
                z = z / math.sqrt(d)
            out[b, h] = z.to(dtype)
    return out


def prefill_inputs(B, H, N, d, dtype=torch.bfloat16, device="cpu", seed=0, dist=None):
    """q, k, v [B,H,N,d] and slopes [H].

    dist "silu": Q,K = SiLU(N(0,1))/sqrt(d), V = N(0,1) (bf16 workloads).
    dist "scaled": Q,K,V = N(0,1)/sqrt(d) (tiny fp32 workload).
    Default: "scaled" for fp32, "silu" otherwise."""
    if dist is None:
        dist = "scaled" if dtype == torch.float32 else "silu"
    g = _gen(seed, device)
    q = _draw((N, d), H, B, g, device, dtype, dist, d)
    k = _draw((N, d), H, B, g, device, dtype, dist, d)
    v = _draw((N, d), H, B, g, device, dtype, "scaled" if dist == "scaled" else "normal", d)
    return q, k, v, slopes(H, device)


def varlen_lengths(num_seqs=16, lo=1024, hi=65536, seed=0):
    """Sequence lengths drawn uniformly from the integers lo..hi inclusive."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randint(lo, hi + 1, (num_seqs,), generator=g).tolist()


def cu_seqlens_of(lengths, device="cpu") -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def varlen_inputs(lengths, H, d, dtype=torch.bfloat16, device="cpu", seed=0, dist=None):
    """Packed q, k, v [H,T,d], cu_seqlens int32 [S+1], slopes [H]."""
    T = int(sum(lengths))
    q, k, v, s = prefill_inputs(1, H, T, d, dtype, device, seed, dist)
    return q[0], k[0], v[0], cu_seqlens_of(lengths, device), s


def decode_inputs(B, H, d, dtype=torch.bfloat16, device="cpu", seed=0, state_sigma=0.01):
    """q, k, v [B,H,d] (SiLU/normal as in the prefill workloads), state [B,H,d,d] fp32."""
    g = _gen(seed, device)
    q = (torch.nn.functional.silu(torch.randn((B, H, d), generator=g, device=device))
         / math.sqrt(d)).to(dtype)
    k = (torch.nn.functional.silu(torch.randn((B, H, d), generator=g, device=device))
         / math.sqrt(d)).to(dtype)
    v = torch.randn((B, H, d), generator=g, device=device).to(dtype)
    state = torch.empty((B, H, d, d), dtype=torch.float32, device=device)
    for b in range(B):
        state[b] = torch.randn((H, d, d), generator=g, device=device) * state_sigma
    return q, k, v, state, slopes(H, device)


def state_inputs(B, H, d, device="cpu", seed=0, sigma=0.5):
    """An incoming state [B,H,d,d] fp32 with entries ~ N(0, sigma^2) (the state of
    a cached prefix; sigma 0.5 is the order of the slow heads' states under the
    prefill workloads' inputs)."""
    g = _gen(seed, device)
    return torch.randn((B, H, d, d), generator=g, device=device) * sigma


def grad_output(shape, dtype=torch.bfloat16, device="cpu", seed=1):
    """dO ~ N(0,1)."""
    g = _gen(seed, device)
    return torch.randn(tuple(shape), generator=g, device=device).to(dtype)
