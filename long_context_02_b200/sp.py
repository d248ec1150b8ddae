"""Sequence parallelism across ranks (LASP+), one process per GPU.

"MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary",
section 3.2: the sequence is cut into consecutive chunks, one per rank. Each
rank summarizes its chunk locally, the summaries are gathered in one
all-gather, and each rank builds its global prefix from them. Here, per rank:

  1. la_prefill_state on the rank's chunk alone gives the chunk's local state
     S_r (keys and values only, no outputs);
  2. one all-gather of the local states (4 MiB per rank at 64 heads, d = 128);
  3. la_state_prefix forms the state before the chunk from the gathered states;
  4. la_prefill_with_state computes the chunk's outputs (and, on the last rank,
     the whole sequence's final state) from that state.

Every arithmetic step runs in the library's kernels; this module only orders
the calls and moves the states between ranks.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import binding as L


def nccl_gather(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """All-gather of one tensor per rank over a torch.distributed process group
    (NCCL for GPUs; any backend that implements all_gather). Returns
    [world, *shape]."""
    import torch.distributed as dist

    def gather(x: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        parts = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(parts, x.contiguous(), group=group)
        return torch.stack(parts)

    return gather


def host_gather(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """All-gather of one tensor per rank staged through host memory, for process
    groups whose backend moves CPU tensors only (gloo): the local state is copied
    to the host, gathered, and the [world, *shape] result copied back to the
    tensor's device."""
    import torch.distributed as dist

    def gather(x: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        xc = x.detach().to("cpu").contiguous()
        parts = [torch.empty_like(xc) for _ in range(world)]
        dist.all_gather(parts, xc, group=group)
        return torch.stack(parts).to(x.device)

    return gather


def local_state(k, v, slopes, ws, stream=None) -> torch.Tensor:
    """Step 1: the state of this rank's chunk alone, [B,H,d,d] fp32."""
    B, H, _, d = k.shape
    st = torch.empty((B, H, d, d), dtype=torch.float32, device=k.device)
    L.la_prefill_state(k, v, slopes, None, st, ws, stream)
    return st


def incoming_state(states, slopes, chunk_lens: Sequence[int], rank: int,
                   stream=None) -> torch.Tensor:
    """Step 3: the state before chunk `rank` from the gathered local states
    [R,B,H,d,d]."""
    R, B, H, d, _ = states.shape
    out = torch.empty((B, H, d, d), dtype=torch.float32, device=states.device)
    L.la_state_prefix(states.contiguous(), slopes, chunk_lens, rank, out, stream)
    return out


def sp_prefill(q, k, v, slopes, chunk_lens: Sequence[int], rank: int, o, state_out,
               gather: Callable[[torch.Tensor], torch.Tensor], ws=None, stream=None):
    """This rank's part of a sequence-parallel prefill.

    q, k, v   [B,H,n_rank,d] on this rank's GPU: chunk `rank` of every sequence
    chunk_lens  host list of every rank's chunk length (n_0, ..., n_{R-1})
    o         [B,H,n_rank,d] out: this chunk's rows of O
    state_out [B,H,d,d] fp32 out (may be None): the state after this chunk,
              which on the last rank is the final state of the whole sequence
    gather    maps this rank's [B,H,d,d] local state to every rank's [R,B,H,d,d]
              (nccl_gather(group) across GPUs); every rank calls it once
    """
    B, H, n, d = q.shape
    if len(chunk_lens) < 1 or chunk_lens[rank] != n:
        raise ValueError("chunk_lens[rank] must equal this rank's chunk length")
    if ws is None:
        ws = L.workspace(L.LA_OP_PREFILL, B, H, n, d, 0, q.dtype, q.device)
    s_loc = local_state(k, v, slopes, ws, stream)
    states = gather(s_loc)
    s_in = incoming_state(states, slopes, chunk_lens, rank, stream)
    L.la_prefill_with_state(q, k, v, slopes, s_in, o, state_out, ws, stream)
