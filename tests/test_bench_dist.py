"""Host logic of bench.py's multi-process path, on CPU with the gloo backend.

Each replica times its own steps; the whole-job number divides the bytes all
ranks processed by the slowest rank's time (max over ranks).  Two processes
on 127.0.0.1 check the barrier, the max-over-ranks reduction, the aggregate,
and that the reference arm does no work on ranks other than 0.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist("gloo")
    bench.barrier()
    ms_local = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms = bench.max_over_ranks(ms_local)
    gbs = bench.whole_job_gbs(1_000_000, 100, world, ms)
    bench.barrier()
    # the reference arm: ranks other than 0 return at once without work
    called = []

    class Args:
        steps, warmup, workload = 1, 3, "msd_small"
    if rank != 0:
        bench.run_reference(Args, bench.get_workload("msd_small"), rank, world)
        called.append("returned")
    out.put((rank, ms, gbs, called))
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, ms, gbs, called in res:
        assert ms == pytest.approx(15.0)                    # max over ranks, identical on both
        assert gbs == pytest.approx(1e6 * 100 * 2 / 15e-3 / 1e9)
    assert res[1][3] == ["returned"]


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_gbs(2_000_000_000, 10, 1, 1000.0) == pytest.approx(20.0)
