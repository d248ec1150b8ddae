"""Run one case of the library a fixed number of times, for profiler captures.

    python -m long_context_02_b200.profile_run CASE [--heads H] [--seq-len N]
           [--segment-tokens S] [--launches K]

CASE is one of
  prefill   la_prefill, bf16 Q/K/V, bf16 O, fp32 final state
  backward  la_backward (three launches each: dQ forward, dK and dV reversed)
  state     la_prefill_state (final state only)
on seeded synthetic inputs of B=1, H heads, N tokens, d=128 (Q, K = SiLU(z)/sqrt(d),
V = N(0,1)). --segment-tokens sets the scan segment length (0 = automatic; a
value above N gives one segment per (head, value half)). Every call goes
through the C ABI; the device status is checked after the last one.
"""
from __future__ import annotations

import argparse

import torch

from . import binding as L
from . import inputs


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["prefill", "backward", "state"])
    ap.add_argument("--heads", type=int, default=64)
    ap.add_argument("--seq-len", type=int, default=8192)
    ap.add_argument("--segment-tokens", type=int, default=0)
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args(argv)
    B, H, N, d = 1, a.heads, a.seq_len, 128
    L.la_set_tuning(0, a.segment_tokens)
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, torch.bfloat16, "cuda", seed=5)
    op = L.LA_OP_BACKWARD if a.case == "backward" else L.LA_OP_PREFILL
    ws = L.workspace(op, B, H, N, d)
    st = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    if a.case == "prefill":
        o = torch.empty_like(q)
        step = lambda: L.la_prefill(q, k, v, s, o, st, ws)
    elif a.case == "state":
        step = lambda: L.la_prefill_state(k, v, s, None, st, ws)
    else:
        do = inputs.grad_output(q.shape, torch.bfloat16, "cuda", seed=6)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        step = lambda: L.la_backward(do, q, k, v, s, dq, dk, dv, ws)
    for _ in range(a.launches):
        step()
    torch.cuda.synchronize()
    status = L.la_read_device_status(ws)
    if status != L.LA_OK:
        raise SystemExit(f"device status {L.la_status_string(status)}")
    print(f"{a.case}: {a.launches} calls of B=1 H={H} N={N} d=128 done")


if __name__ == "__main__":
    main()
