"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the timing
is the maximum over ranks, the value is the whole job's (weak scaling), and the
reference arm runs on rank 0 only."""
import io
import os
import socket
import sys
import contextlib

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local_ms = 10.0 + 5.0 * rank              # rank 1 is the slower one
        bench.barrier(world)
        worst = bench.max_over_ranks(local_ms, world)
        rate = bench.whole_job_rate(8, 200, world, worst)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            class A:                             # reference arm arguments
                workload, steps, warmup, gpus = "tiny-f32-decode", 1, 0, world
            if rank != 0:
                bench.run_reference(A, world, rank)
        out.put((rank, worst, rate, buf.getvalue()))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get() for _ in range(world))
    for rank, worst, rate, printed in res:
        assert worst == pytest.approx(15.0)                       # the slowest rank's time
        assert rate == pytest.approx(2 * 8 * 200 / 0.015)         # both replicas' units
        if rank != 0:
            assert printed == ""                                  # non-zero ranks run no reference arm
