"""Multi-rank host plumbing of bench.py on CPU (gloo, world size 2): every rank
joins the barrier and sees the maximum of the per-rank timings."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist(world, "gloo")
    bench.barrier(dist)
    got = bench.reduce_max(1.5 + rank, dist, torch.device("cpu"))
    out[rank] = got
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=100)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_is_identity():
    import bench

    assert bench.reduce_max(3.25, None, torch.device("cpu")) == 3.25
    bench.barrier(None)
