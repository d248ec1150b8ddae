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

