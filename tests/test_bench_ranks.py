"""The multi-rank logic of bench.py on two CPU ranks (gloo): every rank times its own
independent box (weak scaling, distinct seeds), the job time is the slowest rank's, and the
whole-job value counts every rank's edges.  No GPU is touched."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 3.0 + 2.0 * rank  # rank 1 is the slow one
        t = bench.max_over_ranks(ms, world, dist, torch.device("cpu"))
        out[rank] = (t, bench.rank_seed(2, rank), bench.job_throughput(1000, world, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.0           # both ranks see the slowest rank's time
    assert res[0][1] != res[1][1]                   # independent boxes
    assert res[0][2] == pytest.approx(2 * 1000 / 5e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(4.5, 1) == 4.5
    assert bench.job_throughput(156278, 1, 1.0) == pytest.approx(156278e3)
    assert bench.rank_seed(2, 0) == 2
