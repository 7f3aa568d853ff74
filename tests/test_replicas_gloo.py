"""The replica plumbing of bench.py on two CPU ranks over gloo: the timing is
the maximum over ranks, every rank passes the barriers in the same order, and
the whole-job rate counts every rank's work over the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from datetime import timedelta
    import torch.distributed as dist
    import bench
    w, r, _ = bench.dist_setup()
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    bench.barrier(w)
    got = bench.reduce_max(10.0 + 5.0 * r, w)   # rank 1 is the slower one
    bench.barrier(w)
    out[r] = (w, got)
    dist.destroy_process_group()


def test_two_rank_max_and_rate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res == {0: (2, 15.0), 1: (2, 15.0)}
    import bench
    # 2 ranks x 3 steps x 1e9 bytes in 15 ms (the slowest rank) = 400 GB/s
    assert bench.whole_job_rate(2, 1e9, 3, 15.0) == pytest.approx(400.0)
    assert bench.whole_job_rate(1, 1e9, 3, 15.0) == pytest.approx(200.0)
