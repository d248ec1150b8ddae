"""The multi-rank paths on CPU: two gloo ranks (127.0.0.1).

bench.py runs one replica of the workload per rank (the work shards by
independent heads and sequences, no collective on the data path) and reports
the whole-job rate as all ranks' units over the slowest rank's time. These
tests run that aggregation, and the reference arm's rank rule (rank 0 alone
prints), with world size 2 on the gloo backend. They also run the one
exchange of the sequence-parallel prefill (sp.nccl_gather, the all-gather of
the chunks' local states) and check each rank's incoming state built from
the gathered states against the prefix it stands for.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local_ms = [2.0, 5.0][rank]                  # rank 1 is the slow one
    ms, rate = bench.whole_job_rate(1000, local_ms, world)
    out.put((rank, ms, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_whole_job_rate_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 5.0                          # every rank sees the slowest time
        assert abs(rate - 2 * 1000 / 5e-3) < 1e-6  # both ranks' units over that time


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line(tmp_path):
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--cpu-threads", "2"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _sp_rank_main(rank, world, port, out, which="nccl_gather"):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from long_context_02_b200 import sp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    rng = np.random.default_rng(0)                 # same sequence on every rank
    B, H, d, lens = 1, 2, 4, [5, 9]
    N = sum(lens)
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    lam = np.array([0.6, 0.95])
    a = sum(lens[:rank])
    b = a + lens[rank]
    _, s_loc = oracle.forward(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], lam)
    states = getattr(sp, which)()(torch.from_numpy(s_loc))   # the exchange under test
    s_in = oracle.state_prefix(states.numpy(), lam, lens, rank)
    _, want = oracle.forward(q[:, :, :a], k[:, :, :a], v[:, :, :a], lam)
    ok = tuple(states.shape) == (world, B, H, d, d) and np.allclose(s_in, want, rtol=1e-12,
                                                                    atol=1e-12)
    out.put((rank, bool(ok)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("which", ["nccl_gather", "host_gather"])
def test_sequence_parallel_exchange_two_ranks(which):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sp_rank_main, args=(r, 2, port, q, which)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, True), (1, True)]
