"""The N > 1 host path of bench.py on host cores: two gloo ranks, as
torch.distributed.run would start them.  The data path has no collective;
what the ranks share is the barrier and the max over ranks of each timing,
from which the whole-job (weak-scaling) throughput is formed."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    ctx = bench.DistCtx(world, backend="gloo")
    try:
        ctx.barrier()
        ms = [12.0, 20.0][rank]                   # rank 1 is the slower one
        rate, t = ctx.job_rate(1000.0, ms)
        q.put((rank, ctx.world, ctx.max(float(rank)), rate, t))
        ctx.barrier()
    finally:
        ctx.close()


def test_two_gloo_ranks_take_the_slowest_rank_for_the_job():
    world, port = 2, _free_port()
    smp = mp.get_context("spawn")
    q = smp.Queue()
    procs = [smp.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, mx, rate, t in got:
        assert w == 2
        assert mx == 1.0                           # max over ranks, seen by every rank
        assert t == 20.0                           # the job lasts as long as its slowest rank
        assert rate == pytest.approx(2 * 1000.0 / 0.020)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    ctx = bench.DistCtx(1, backend="gloo")
    assert not ctx.on
    rate, t = ctx.job_rate(500.0, 10.0)
    assert t == 10.0 and rate == pytest.approx(500.0 / 0.010)
    ctx.close()
