"""bench.py's conventions and bookkeeping on CPU: the FLOP and byte counts of
the MiniMax-shaped workload, and the rule that the profiled DRAM traffic is
only reported for the kernel source it was captured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_flop_and_byte_conventions():
    # B*H*N*(4d^2 + 4*256*d) at B=1, H=64, N=32768, d=128
    assert bench.prefill_flops(1, 64, 32768) == 64 * 32768 * (4 * 128 * 128 + 4 * 256 * 128)
    assert abs(bench.prefill_flops(1, 64, 32768) - 4.123e11) / 4.123e11 < 1e-3
    # Q, K, V read and O written once (bf16) plus the fp32 final state
    assert bench.prefill_bytes(1, 64, 32768) == 4 * 64 * 32768 * 128 * 2 + 64 * 128 * 128 * 4


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    prof = tmp_path / "p.txt"
    prof.write_text(f"# summary\nkernel_source_sha256_16: {bench.kernel_source_hash()}\n"
                    "dram_bytes_per_full_launch: 123456\n")
    monkeypatch.setattr(bench, "PROFILE", str(prof))
    assert bench.profiled_traffic() == 123456.0
    prof.write_text("kernel_source_sha256_16: 0000000000000000\ndram_bytes_per_full_launch: 1\n")
    assert bench.profiled_traffic() is None



def test_quadratic_form_sample_extrapolates_by_the_row_costs():
    """The CPU baseline's quadratic-form leg: a sample of rows, scaled to the
    whole workload by the number of (i+1) terms (here one head, rows 4095,
    8191, ..., 32767)."""
    import numpy as np
    import torch

    import oracle
    from long_context_02_b200 import inputs
    q, k, v, _ = inputs.prefill_inputs(1, 1, bench.N_, bench.D_, torch.bfloat16, "cpu", seed=0)
    f = lambda t: t.to(torch.float64).numpy()
    r = bench.cpu_quadratic_sample(f(q), f(k), f(v), oracle.default(), 1, n_heads=1,
                                   stride=4096)
    rows = np.arange(4095, bench.N_, 4096)
    ratio = 64 * bench.N_ * (bench.N_ + 1) / 2 / float(np.sum(rows + 1))
    t_sample = r["extrapolated_s"] / ratio
    assert r["value"] > 0 and r["extrapolated_s"] > 0
    want = bench.prefill_flops(1, 64, bench.N_) / (t_sample * ratio) / 1e12
    assert abs(r["value"] - want) <= 1e-3 * want  # both figures are rounded in the report


def test_clock_sampler_counts_only_samples_inside_the_timed_loop():
    """bench.ClockSampler reports the clocks of the samples taken while the
    timed loop ran (the window timed() marks), not the idle GPU around it."""
    import threading
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = [(0.0, 1965.0, 1965.0, 0x1, 200.0),     # idle, before
                 (1.0, 1600.0, 1965.0, 0x4, 990.0),     # under load, power cap
                 (1.5, 1650.0, 1965.0, 0x4, 1001.0),
                 (3.0, 1965.0, 1965.0, 0x1, 250.0)]     # idle, after
    s.window = [0.9, 2.0]
    s.thread = threading.Thread(target=lambda: None)
    s.thread.start()
    s.stop_flag = False
    s.proc = None
    r = s.stop()
    assert r["under_load"] and r["samples"] == 2
    assert r["sm_mhz"] == 1625.0 and r["sm_mhz_min"] == 1600.0
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 1001.0
