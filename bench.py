#!/usr/bin/env python
"""Benchmark of lightning attention on B200 (one JSON line on rank 0).

Headline step: one prefill (la_prefill) of the MiniMax-shaped workload,
B=1, H=64, N=32768, d=128, bf16 Q/K/V (Q,K = SiLU(N(0,1))/sqrt(d), V = N(0,1),
slopes 2^(-8(h+1)/H)), bf16 O and fp32 final state, inputs resident in HBM.
The three input tensors (1.5 GB) exceed the 126 MB L2, so no flush is needed
between steps.

FLOP convention (fixed, algorithmic): per token and head 4 d^2 + 4 * 256 * d,
the pages' O(n d^2 + n B d) complexity with their base tile of 256
("MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary",
sections 2.2 and 3.3). Algorithmic bytes: Q, K, V read once, O written once,
plus the final fp32 state.

Other legs in the same line: `e2e` (host buffers, copies inside the timed
region), `roofline` (HBM), `cpu_baseline` (the fp64 oracle on the host cores,
bounded sample), and `secondary` measurements (decode, backward, varlen,
long context). Multi-GPU (torchrun): every rank runs its own replica of the
workload (the path shards by independent heads/sequences, no collective on
the data path); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only other implementation the
sources allow) on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "lightning-attn prefill TFLOP/s & tokens/s (H=64,d=128) + % tensor peak; decode GB/s"
B_, H_, N_, D_ = 1, 64, 32768, 128
FLOP_PER_TOKEN_HEAD = 4 * D_ * D_ + 4 * 256 * D_            # 196,608
FLOP_PER_TOKEN_HEAD_BWD = 10 * D_ * D_ + 10 * 256 * D_
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE = os.path.join(ROOT, "profiles", "tc_forward_kernel.minimax_prefill_32k.txt")
KERNEL_SRC = os.path.join(ROOT, "long_context_02_b200", "csrc", "tc_forward.cu")


def prefill_flops(B, H, N):
    return B * H * N * FLOP_PER_TOKEN_HEAD


def prefill_bytes(B, H, N, d=D_, out_bytes=2):
    return B * H * N * d * (3 * 2 + out_bytes) + B * H * d * d * 4


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return PEAKS_FALLBACK, "fallback"


def kernel_source_hash():
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic():
    """Per-launch DRAM traffic of the prefill kernel from the committed ncu summary,
    or None when the kernel source changed since those counters were taken."""
    if not os.path.exists(PROFILE):
        return None
    vals = {}
    with open(PROFILE) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    try:
        if vals.get("kernel_source_sha256_16") != kernel_source_hash():
            return None
        return float(vals["dram_bytes_per_full_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event reasons while the timed loop runs.

    Sampled through NVML (the library nvidia-smi reports from) every ~1 ms in a
    background thread; only samples inside the window that timed() marks with
    begin()/end() count as "under load". The timed region is short (20 prefill
    steps take ~12 ms), so a sampler at nvidia-smi's 50 ms period would mostly
    see the idle GPU around it. Falls back to nvidia-smi samples when NVML is
    unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device):
        self.samples = []
        self.window = None
        self.thread = None
        self.proc = None
        self.nvml = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu = str(device)
        self.err = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(self.gpu)
            self.nvml = pynvml
        except Exception as e:  # noqa: BLE001 - any NVML failure selects the fallback
            self.nvml = None
            self.err = f"nvml: {type(e).__name__}: {e}"[:200]

    def _run(self):
        n = self.nvml
        max_mhz = 0.0
        while not self.stop_flag:
            try:
                if not max_mhz:
                    max_mhz = n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM)
                mhz = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                watts = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                self.samples.append((time.perf_counter(), float(mhz), float(max_mhz), int(reasons),
                                     watts))
            except Exception as e:  # noqa: BLE001
                self.err = f"nvml sample: {type(e).__name__}: {e}"[:200]
            time.sleep(0.001)

    def start(self):
        import threading
        self.samples, self.window = [], None
        if self.nvml is not None:
            self.stop_flag = False
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            time.sleep(0.01)
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            fields = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                      "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                      "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={fields}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def _snapshot(self):
        """One nvidia-smi reading, when no sample could be taken in the loop."""
        try:
            out = subprocess.run(
                ["nvidia-smi", "-i", self.gpu, "--query-gpu=clocks.sm,clocks.max.sm,"
                 "clocks_event_reasons.sw_power_cap", "--format=csv,noheader,nounits"],
                capture_output=True, text=True, timeout=10).stdout.strip().split(",")
            return {"sm_mhz": float(out[0]), "sm_max_mhz": float(out[1]),
                    "reasons": ["sw_power_cap"] if "active" in out[2].lower() else [],
                    "samples": 1, "under_load": False, "source": "nvidia-smi, one reading after"}
        except Exception as e:  # noqa: BLE001
            return {"error": (self.err or "") + f"; nvidia-smi: {type(e).__name__}: {e}"[:200]}

    def begin(self):
        self.window = [time.perf_counter(), None]

    def end(self):
        if self.window is not None and self.window[1] is None:
            self.window[1] = time.perf_counter()

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            rows = self.samples
            if self.window and self.window[1] is not None:
                inside = [r for r in rows if self.window[0] <= r[0] <= self.window[1]]
            else:
                inside = []
            use = inside or rows
            if not use:
                return self._snapshot()
            reasons = sorted({name for r in use for name, bit in self.REASONS if r[3] & bit})
            return {"sm_mhz": statistics.median(r[1] for r in use),
                    "sm_mhz_min": min(r[1] for r in use),
                    "sm_max_mhz": max(r[2] for r in use), "reasons": reasons,
                    "power_w_max": round(max(r[4] for r in use), 1),
                    "samples": len(use), "under_load": bool(inside), "source": "nvml, 1 ms"}
        if self.proc is None:
            return self._snapshot()
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[4:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return self._snapshot()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(1, 5)
                          if r[i].lower() in ("active", "1", "yes")})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "under_load": False, "source": "nvidia-smi, 50 ms"}


# ---------------------------------------------------------------- distributed

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank scalar over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, local_ms, world):
    """Aggregate throughput of `world` replicas: all units over the slowest rank's time.
    Returns (max ms over ranks, units per second)."""
    ms = max_over_ranks(local_ms, world)
    return ms, world * units_per_rank / (ms * 1e-3)


def timed(fn, steps, world, stream=None, sampler=None):
    """Device time of `steps` calls of fn (ms per step), max over ranks. A clock
    sampler, if given, counts only the samples taken while the loop runs."""
    stream = stream or torch.cuda.current_stream()
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    if sampler is not None:
        sampler.begin()
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.end()
    barrier(world)
    return max_over_ranks(a.elapsed_time(b) / steps, world)


# ---------------------------------------------------------------- our arm

def run_ours(args):
    from long_context_02_b200 import binding as L
    from long_context_02_b200 import inputs

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    L.lib()  # fails loudly when the library is missing
    pk, pk_kind = peaks()
    N = args.seq_len

    q, k, v, s = inputs.prefill_inputs(B_, H_, N, D_, torch.bfloat16, dev, seed=1000 + rank)
    o = torch.empty_like(q)
    st = torch.empty((B_, H_, D_, D_), dtype=torch.float32, device=dev)
    ws = L.workspace(L.LA_OP_PREFILL, B_, H_, N, D_, 0, torch.bfloat16, dev)

    def step():
        L.la_prefill(q, k, v, s, o, st, ws)

    for _ in range(max(args.warmup, 3)):
        step()
    assert L.la_read_device_status(ws) == L.LA_OK
    launches_per_step = L.la_last_launch_count()
    sampler = ClockSampler(dev)
    sampler.start()
    ms = timed(step, args.steps, world, sampler=sampler)
    clocks = sampler.stop()
    assert L.la_read_device_status(ws) == L.LA_OK

    F = prefill_flops(B_, H_, N)
    Bytes = prefill_bytes(B_, H_, N)
    value = world * F / (ms * 1e-3) / 1e12  # ms is already the max over ranks
    achieved = Bytes / (ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                "traffic": profiled_traffic() if N == N_ else None, "peak_source": pk_kind,
                "kernel": "tc_forward_kernel", "algorithmic_bytes": Bytes}

    # End to end through the C ABI with host buffers: H2D of Q,K,V from pinned
    # memory, the calls, D2H of O and the state, all inside the timed region.
    # The heads are processed in groups on three streams (copy in, compute,
    # copy out), so one group's copies overlap another group's prefill: the
    # way a caller holding host tensors would drive the library.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hst = torch.empty(st.shape, dtype=st.dtype).pin_memory()
        groups = 8
        hg = H_ // groups
        ws_g = L.workspace(L.LA_OP_PREFILL, B_, hg, N, D_, 0, torch.bfloat16, dev)
        s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))

        def e2e_step():
            cur = torch.cuda.current_stream()
            s_in.wait_stream(cur)
            for g in range(groups):
                h = slice(g * hg, (g + 1) * hg)
                with torch.cuda.stream(s_in):
                    for dst, src in ((q, hq), (k, hk), (v, hv)):
                        dst[:, h].copy_(src[:, h], non_blocking=True)
                    loaded = s_in.record_event()
                s_cmp.wait_event(loaded)
                L.la_prefill(q[:, h], k[:, h], v[:, h], s[h], o[:, h], st[:, h], ws_g, stream=s_cmp)
                done = s_cmp.record_event()
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    ho[:, h].copy_(o[:, h], non_blocking=True)
                    hst[:, h].copy_(st[:, h], non_blocking=True)
            cur.wait_stream(s_out)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        assert L.la_read_device_status(ws_g) == L.LA_OK
        e2e_steps = max(2, min(args.steps, 20))
        ms_e2e = timed(e2e_step, e2e_steps, world)
        h2d = 3 * q.numel() * q.element_size()
        d2h = o.numel() * o.element_size() + st.numel() * 4
        e2e = {"value": round(world * F / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "ms_per_step": round(ms_e2e, 4), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "schedule": f"{groups} head groups, copy-in / prefill / copy-out on 3 streams"}
        del hq, hk, hv, ho, hst

    secondary = {} if args.no_secondary else run_secondary(args, L, inputs, dev, world, pk, rank)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.cpu_heads, args.cpu_threads)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: Q,K = SiLU(N(0,1))/sqrt(d), V = N(0,1))",
        "config": {"workload": f"MiniMax-shaped prefill B=1 H=64 N={N} d=128 bf16",
                   "B": B_, "H": H_, "N": N, "d": D_, "global_batch": B_ * world,
                   "seq_len": N, "out_dtype": "bf16", "state": "fp32",
                   "parallelism": f"replicas x{world} (independent heads, no collective)",
                   "l2": (f"inputs ({3 * q.numel() * 2 / 1e9:.2f} GB per step) larger than the "
                          "126 MB L2; no flush"),
                   "flop_convention": "B*H*N*(4d^2 + 4*256*d)"},
        "tokens_per_s": round(world * B_ * N / (ms * 1e-3), 1),
        "token_heads_per_s": round(world * B_ * H_ * N / (ms * 1e-3), 1),
        "pct_tensor_peak": round(100 * value / world / pk["bf16_tflops"], 2),
        "tflops_executed": round(world * B_ * H_ * N * (4 * D_ * D_ * 1.25 + 4 * 128 * D_)
                                 / (ms * 1e-3) / 1e12, 3),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "secondary": secondary,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_mixed(L, inputs, dev, world, steps):
    """A batch of 20 cached inputs, two of 50 tokens and 18 of one token (the
    shape of the separated prefill/decode example in section 3.3 of the
    MiniMax-01 summary), H=64, d=128: la_mixed_step with prefill and decode on
    two streams, on one stream, and the whole batch through the prefill kernel."""
    lengths = [1] * 20
    lengths[3] = lengths[11] = 50
    H, d, S = 64, 128, len(lengths)
    q, k, v, cu, s = inputs.varlen_inputs(lengths, H, d, torch.bfloat16, dev, seed=17)
    T = q.shape[1]
    st = inputs.state_inputs(S, H, d, dev, seed=18)
    o = torch.empty_like(q)
    ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, H, T, d, S, torch.bfloat16, dev)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=dev)

    def two():
        side.wait_stream(main)
        L.la_mixed_step(cu, q, k, v, s, st, o, ws, main, side)
        main.wait_stream(side)

    legs = {"two_streams": two,
            "one_stream": lambda: L.la_mixed_step(cu, q, k, v, s, st, o, ws, main, main),
            "prefill_kernel_only":
                lambda: L.la_prefill_varlen_with_state(cu, q, k, v, s, st, o, st, ws)}
    res = {"workload": "20 cached inputs (2 x 50 tokens, 18 x 1 token) H=64 d=128 bf16, "
                       "fp32 states advanced in place"}
    n = max(20, steps)
    for name, fn in legs.items():
        for _ in range(3):
            fn()
        res[name + "_us"] = round(1e3 * timed(fn, n, world), 2)
    del q, k, v, st, o, ws
    return res


def bench_sp(L, inputs, dev, world, rank, steps):
    """One MiniMax-shaped sequence (B=1, H=64, N=32768, d=128, bf16) cut into
    `world` consecutive chunks, one per rank: every rank runs sp.sp_prefill on
    its chunk with the NCCL all-gather of the local states (4 MiB per rank)
    inside the timed region. The rate is the whole sequence's FLOPs over the
    slowest rank's time (strong scaling of one sequence)."""
    from long_context_02_b200 import sp
    n = N_ // world
    q, k, v, s = inputs.prefill_inputs(1, H_, N_, D_, torch.bfloat16, dev, seed=19)
    qc, kc, vc = (t[:, :, rank * n:(rank + 1) * n].contiguous() for t in (q, k, v))
    del q, k, v
    o = torch.empty_like(qc)
    st = torch.empty((1, H_, D_, D_), dtype=torch.float32, device=dev)
    ws = L.workspace(L.LA_OP_PREFILL, 1, H_, n, D_, 0, torch.bfloat16, dev)
    gather = sp.nccl_gather()
    fn = lambda: sp.sp_prefill(qc, kc, vc, s, [n] * world, rank, o, st, gather, ws)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    assert L.la_read_device_status(ws) == L.LA_OK
    ms = timed(fn, steps, world)
    F = prefill_flops(1, H_, N_)
    res = {"workload": f"sequence-parallel prefill of one B=1 H=64 N={N_} d=128 bf16 sequence "
                       f"over {world} ranks ({n}-token chunks); local state, NCCL all-gather "
                       "of the local states, prefix, prefill from it: all timed",
           "ms": round(ms, 4), "TFLOP/s": round(F / (ms * 1e-3) / 1e12, 2),
           "tokens_per_s": round(N_ / (ms * 1e-3), 1), "scaling": "strong"}
    del qc, kc, vc, o, st, ws
    return res


def run_secondary(args, L, inputs, dev, world, pk, rank=0):
    out = {}
    steps = max(3, min(args.steps, 50))
    # decode: batch 256, H=64, d=128, fp32 state [256,64,128,128] ~ N(0, 0.01)
    qd, kd, vd, state, sd = inputs.decode_inputs(256, 64, 128, torch.bfloat16, dev, seed=7)
    od = torch.empty_like(qd)
    fn = lambda: L.la_decode(qd, kd, vd, sd, state, od)
    for _ in range(3):
        fn()
    ms = timed(fn, steps, world)
    nbytes = 2 * state.numel() * 4 + 4 * qd.numel() * 2
    out["decode"] = {"workload": "decode B=256 H=64 d=128 bf16, fp32 state 1 GiB",
                     "ms": round(ms, 4), "GB/s": round(world * nbytes / (ms * 1e-3) / 1e9, 1),
                     "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                     "bytes": nbytes}
    del qd, kd, vd, state, od
    # backward: config-2 shape
    q, k, v, s = inputs.prefill_inputs(1, 64, 32768, 128, torch.bfloat16, dev, seed=11)
    do = inputs.grad_output(q.shape, torch.bfloat16, dev, seed=12)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = L.workspace(L.LA_OP_BACKWARD, 1, 64, 32768, 128, 0, torch.bfloat16, dev)
    fn = lambda: L.la_backward(do, q, k, v, s, dq, dk, dv, ws)
    for _ in range(3):
        fn()
    ms = timed(fn, max(3, steps // 5), world)
    F = 1 * 64 * 32768 * FLOP_PER_TOKEN_HEAD_BWD
    nbytes = 7 * q.numel() * 2
    out["backward"] = {"workload": "backward B=1 H=64 N=32768 d=128 bf16",
                       "ms": round(ms, 4), "TFLOP/s": round(world * F / (ms * 1e-3) / 1e12, 2),
                       "GB/s_algorithmic": round(nbytes / (ms * 1e-3) / 1e9, 1),
                       "flop_convention": "B*H*N*(10d^2 + 10*256*d)"}
    del q, k, v, do, dq, dk, dv, ws
    # prefill continued from a cached prefix's state (state advanced in place)
    q, k, v, s = inputs.prefill_inputs(1, 64, 32768, 128, torch.bfloat16, dev, seed=15)
    st = inputs.state_inputs(1, 64, 128, dev, seed=16)
    o = torch.empty_like(q)
    ws = L.workspace(L.LA_OP_PREFILL, 1, 64, 32768, 128, 0, torch.bfloat16, dev)
    fn = lambda: L.la_prefill_with_state(q, k, v, s, st, o, st, ws)
    for _ in range(3):
        fn()
    ms = timed(fn, steps, world)
    F = prefill_flops(1, 64, 32768)
    nbytes = prefill_bytes(1, 64, 32768) + st.numel() * 4
    out["prefill_with_state"] = {
        "workload": "prefill from a cached prefix's state B=1 H=64 N=32768 d=128 bf16, "
                    "state in place",
        "ms": round(ms, 4), "TFLOP/s": round(world * F / (ms * 1e-3) / 1e12, 2),
        "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
    del q, k, v, st, o, ws
    # final state alone (a prefix to cache, or a chunk's local state): K, V in, state out
    q, k, v, s = inputs.prefill_inputs(1, 64, 32768, 128, torch.bfloat16, dev, seed=21)
    del q
    st = torch.empty((1, 64, 128, 128), dtype=torch.float32, device=dev)
    ws = L.workspace(L.LA_OP_PREFILL, 1, 64, 32768, 128, 0, torch.bfloat16, dev)
    fn = lambda: L.la_prefill_state(k, v, s, None, st, ws)
    for _ in range(3):
        fn()
    ms = timed(fn, steps, world)
    nbytes = 2 * k.numel() * 2 + st.numel() * 4
    out["prefill_state_only"] = {
        "workload": "final state only, B=1 H=64 N=32768 d=128 bf16 (K, V in; state out)",
        "ms": round(ms, 4), "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
        "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
    del k, v, st, ws
    out["mixed"] = bench_mixed(L, inputs, dev, world, steps)
    # one rank's step of a sequence-parallel prefill: the 32K x 64 workload cut into
    # 8 chunks of 4096 tokens, the last rank's chunk; the gather returns the
    # already-gathered states (the NCCL all-gather of 8 x 4 MiB is not timed here)
    from long_context_02_b200 import sp
    R, n = 8, 32768 // 8
    q, k, v, s = inputs.prefill_inputs(1, 64, n, 128, torch.bfloat16, dev, seed=19)
    o = torch.empty_like(q)
    st = torch.empty((1, 64, 128, 128), dtype=torch.float32, device=dev)
    states = inputs.state_inputs(R, 64, 128, dev, seed=20).reshape(R, 1, 64, 128, 128)
    ws = L.workspace(L.LA_OP_PREFILL, 1, 64, n, 128, 0, torch.bfloat16, dev)
    fn = lambda: sp.sp_prefill(q, k, v, s, [n] * R, R - 1, o, st, lambda _: states, ws)
    for _ in range(3):
        fn()
    ms = timed(fn, steps, world)
    out["sp_rank_step"] = {
        "workload": "sequence-parallel prefill, one rank of 8: 4096-token chunk of the "
                    "H=64 d=128 bf16 32K workload (local prefill, prefix of 8 states, "
                    "prefill from that state; all-gather not included)",
        "ms": round(ms, 4)}
    del q, k, v, o, st, states, ws
    if world > 1:
        out["sp"] = bench_sp(L, inputs, dev, world, rank, steps)
    # output normalization and gate on the prefill's output (bf16 O, gate and Y)
    o = torch.randn((1, 64, 32768, 128), device=dev).to(torch.bfloat16)
    g = torch.randn((1, 32768, 64 * 128), device=dev).to(torch.bfloat16)
    w = torch.ones(64 * 128, device=dev)
    y = torch.empty_like(g)
    fn = lambda: L.la_output_norm_gate(o, g, w, 1e-5, y)
    for _ in range(3):
        fn()
    ms = timed(fn, steps, world)
    nbytes = 3 * o.numel() * 2
    out["norm_gate"] = {"workload": "RMS norm over H*d + sigmoid gate, B=1 H=64 N=32768 d=128 bf16",
                        "ms": round(ms, 4), "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                        "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                        "bytes": nbytes}
    del o, g, w, y
    if not args.quick:
        # varlen: 16 sequences of U{1024..65536} tokens, packed
        lengths = inputs.varlen_lengths(16, 1024, 65536, seed=0)
        qv, kv, vv, cu, sv = inputs.varlen_inputs(lengths, 64, 128, torch.bfloat16, dev, seed=13)
        T = int(sum(lengths))
        ov = torch.empty_like(qv)
        stv = torch.empty((16, 64, 128, 128), dtype=torch.float32, device=dev)
        ws = L.workspace(L.LA_OP_PREFILL_VARLEN, 1, 64, T, 128, 16, torch.bfloat16, dev)
        fn = lambda: L.la_prefill_varlen(cu, qv, kv, vv, sv, ov, stv, ws)
        for _ in range(3):
            fn()
        ms = timed(fn, max(3, steps // 5), world)
        F = T * 64 * FLOP_PER_TOKEN_HEAD
        nbytes = prefill_bytes(1, 64, T) + (16 - 1) * 64 * 128 * 128 * 4
        out["varlen"] = {"workload": f"varlen 16 seqs U{{1024..65536}} (T={T}) H=64 d=128 bf16",
                         "ms": round(ms, 4), "TFLOP/s": round(world * F / (ms * 1e-3) / 1e12, 2),
                         "tokens_per_s": round(world * T / (ms * 1e-3), 1),
                         "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        del qv, kv, vv, ov, stv, ws
        # long context: N = 1,048,576 (Q, K, V, O ~16 GB each)
        NL = 1 << 20
        q, k, v, s = inputs.prefill_inputs(1, 64, NL, 128, torch.bfloat16, dev, seed=14)
        o = torch.empty_like(q)
        st = torch.empty((1, 64, 128, 128), dtype=torch.float32, device=dev)
        ws = L.workspace(L.LA_OP_PREFILL, 1, 64, NL, 128, 0, torch.bfloat16, dev)
        fn = lambda: L.la_prefill(q, k, v, s, o, st, ws)
        for _ in range(3):
            fn()
        ms = timed(fn, 3, world)
        F = prefill_flops(1, 64, NL)
        nbytes = prefill_bytes(1, 64, NL)
        out["long"] = {"workload": "long prefill B=1 H=64 N=1048576 d=128 bf16",
                       "ms": round(ms, 3), "TFLOP/s": round(world * F / (ms * 1e-3) / 1e12, 2),
                       "tokens_per_s": round(world * NL / (ms * 1e-3), 1),
                       "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}
        del q, k, v, o, st, ws
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- CPU oracle

def cpu_threads_used(requested=None):
    n = len(os.sched_getaffinity(0))
    return min(n, requested) if requested else n


def cpu_baseline(n_heads=64, threads=None, seed=0):
    """The fp64 oracle as it stands (token recurrence, O(N d^2) per head) on the
    headline workload, or a bounded sample of it: n_heads of the 64 heads (all
    of them by default, a few seconds on 16 cores), all 32768 tokens. Reported
    in the headline unit (FLOP convention above)."""
    import oracle
    from long_context_02_b200 import inputs
    th = cpu_threads_used(threads)
    os.environ["OMP_NUM_THREADS"] = str(th)
    q, k, v, s = inputs.prefill_inputs(1, n_heads, N_, D_, torch.bfloat16, "cpu", seed=seed)
    s = inputs.slopes(H_)[:n_heads]
    lam = oracle.lambdas_from_slopes(s.numpy())
    f = lambda t: t.to(torch.float64).numpy()
    qn, kn, vn = f(q), f(k), f(v)
    orc = oracle.default()
    t0 = time.perf_counter()
    orc.recurrence(qn, kn, vn, lam)
    dt = time.perf_counter() - t0
    F = prefill_flops(1, n_heads, N_)
    return {"value": round(F / dt / 1e12, 6), "unit": "TFLOP/s", "cores": th, "kind": "oracle",
            "sample": f"fp64 token recurrence on {n_heads} of 64 heads x {N_} tokens, d=128 "
                      f"({dt:.1f} s)",
            "tokens_per_s": round(N_ * n_heads / 64 / dt, 1),
            "quadratic_form": cpu_quadratic_sample(qn, kn, vn, orc, th)}


def cpu_quadratic_sample(qn, kn, vn, orc, threads, n_heads=8, stride=16):
    """The oracle's quadratic form (the operator's definition, O(N^2 d) per head)
    timed on a labelled sample of the headline workload and extrapolated to the
    whole of it. Sample: rows i = stride-1, 2*stride-1, ..., N-1 of n_heads heads
    (data of the first heads, decays of heads spread over 0..63). Row i costs
    (i+1) terms, so the whole workload's time is the sample's time times
    64 * N(N+1)/2 over the sample's sum of (i+1)."""
    import numpy as np

    import oracle
    from long_context_02_b200 import inputs
    lam_all = oracle.lambdas_from_slopes(inputs.slopes(H_).numpy())
    heads = [round(x) for x in np.linspace(0, H_ - 1, n_heads)]
    rows = np.arange(stride - 1, N_, stride, dtype=np.int64)
    n_heads = min(n_heads, qn.shape[1])
    t0 = time.perf_counter()
    for i in range(n_heads):
        orc.forward_rows(qn[0, i], kn[0, i], vn[0, i], lam_all[heads[i]], rows)
    dt = time.perf_counter() - t0
    terms_sample = n_heads * float(np.sum(rows + 1))
    terms_full = H_ * N_ * (N_ + 1) / 2.0
    t_full = dt * terms_full / terms_sample
    F = prefill_flops(1, H_, N_)
    return {"value": round(F / t_full / 1e12, 8), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle (quadratic form)",
            "sample": f"quadratic-form rows {stride - 1}, {2 * stride - 1}, ..., {N_ - 1} "
                      f"({len(rows)} rows) of {n_heads} heads (decays of heads {heads}), "
                      f"{dt:.1f} s",
            "extrapolated_s": round(t_full, 1),
            "extrapolation": "t_full = t_sample * (64 * N(N+1)/2) / (sum over sampled "
                             "(head, row i) of (i+1))"}


def run_reference(args):
    """The oracle on the host cores, same metric/unit/config, bounded samples."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np  # noqa: F401

    import oracle
    from long_context_02_b200 import inputs
    th = cpu_threads_used(args.cpu_threads)
    os.environ["OMP_NUM_THREADS"] = str(th)
    n_heads = min(H_, max(1, th))
    # each step: the first n_tok tokens of n_heads heads (about 0.1 s on 16
    # cores at the default 4096), so that --steps 200 still ends in well under
    # a minute; the rate per FLOP does not depend on the sample
    n_tok = max(128, min(N_, args.ref_tokens))
    q, k, v, _ = inputs.prefill_inputs(1, n_heads, n_tok, D_, torch.bfloat16, "cpu", seed=0)
    lam = oracle.lambdas_from_slopes(inputs.slopes(H_)[:n_heads].numpy())
    f = lambda t: t.to(torch.float64).numpy()
    qn, kn, vn = f(q), f(k), f(v)
    orc = oracle.default()
    for _ in range(args.warmup):
        orc.recurrence(qn[:, :, :128], kn[:, :, :128], vn[:, :, :128], lam)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.recurrence(qn, kn, vn, lam)
    dt = (time.perf_counter() - t0) / args.steps
    F = prefill_flops(1, n_heads, n_tok)
    value = F / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "MiniMax-shaped prefill B=1 H=64 N=32768 d=128 bf16",
                       "B": B_, "H": H_, "N": N_, "d": D_,
                       "flop_convention": "B*H*N*(4d^2 + 4*256*d)"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": th,
                             "kind": "oracle",
                             "sample": f"each step: fp64 token recurrence on {n_heads} of 64 "
                                       f"heads x the first {n_tok} of {N_} tokens"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="skip the varlen and long legs")
    ap.add_argument("--seq-len", type=int, default=N_,
                    help="tokens of the headline prefill (default: the MiniMax-shaped 32768)")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-heads", type=int, default=64)
    ap.add_argument("--cpu-threads", type=int, default=0)
    ap.add_argument("--ref-tokens", type=int, default=4096,
                    help="tokens per head in each step of the reference (oracle) arm")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
