"""The sequence-parallel prefill (LASP+) as separate processes: two ranks, each
its own process with its own CUDA context on cuda:0, exchanging their chunks'
local states through a gloo process group on 127.0.0.1.

"MiniMax-01: Scaling Foundation Models with Lightning Attention | Summary",
section 3.2: each partition summarizes its chunk, one all-gather shares the
summaries, and each partition builds its global prefix from them. Here every
rank runs long_context_02_b200.sp.sp_prefill around the library's kernels with
a real collective (sp.host_gather: the local state staged through host memory,
gathered over gloo). No kernel waits on another rank: the only exchange is the
host-side all-gather between the two kernel sequences, so running both
processes on one GPU is safe. Every rank's rows and the last rank's final state
are compared with the fp64 oracle on the whole sequence.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from long_context_02_b200 import inputs
from tests.gpu_util import TOL_BF16, TOL_F32, assert_close, f64, lam

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, shape, dtype, lens, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from long_context_02_b200 import binding as L
    from long_context_02_b200 import inputs as inp
    from long_context_02_b200 import sp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        L.la_set_tuning(64 if dtype == torch.float32 else 0, 0)
        B, H, N, d = shape
        q, k, v, s = inp.prefill_inputs(B, H, N, d, dtype, "cuda", seed=41)  # same on every rank
        a = sum(lens[:rank])
        b = a + lens[rank]
        qc, kc, vc = (t[:, :, a:b].contiguous() for t in (q, k, v))
        o = torch.empty(qc.shape, dtype=torch.float32, device="cuda")
        st = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
        sp.sp_prefill(qc, kc, vc, s, lens, rank, o, st, gather=sp.host_gather())
        torch.cuda.synchronize()
        out.put((rank, o.cpu().numpy(), st.cpu().numpy()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,shape,lens,tol", [
    (torch.bfloat16, (1, 4, 3000, 128), [1300, 1700], TOL_BF16),   # tensor-core path
    (torch.float32, (2, 2, 700, 64), [129, 571], TOL_F32),         # fp32 path
])
def test_sequence_parallel_prefill_two_processes(dtype, shape, lens, tol):
    world = len(lens)
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, shape, dtype, lens, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = dict((r, (o, st)) for r, o, st in (q_out.get(timeout=300) for _ in range(world)))
    finally:
        for p in procs:
            p.join(timeout=120)
    for p in procs:
        assert p.exitcode == 0
    B, H, N, d = shape
    q, k, v, s = inputs.prefill_inputs(B, H, N, d, dtype, "cuda", seed=41)
    o_ref, st_ref = oracle.forward(f64(q), f64(k), f64(v), lam(s))
    a = 0
    for r in range(world):
        b = a + lens[r]
        assert_close(res[r][0], o_ref[:, :, a:b], tol, f"rank {r} rows")
        a = b
    assert_close(res[world - 1][1], st_ref, tol, "final state on the last rank")
