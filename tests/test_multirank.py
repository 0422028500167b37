"""Multi-rank host logic of bench.py on CPU (gloo, world_size 2): the
max-over-ranks timing reduction and per-rank replicas of the workload."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    import workloads as W

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_info()
        assert (w, r) == (world, rank)
        # each rank reports its own time; everyone gets the max
        mx = bench.reduce_max(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        # replicas draw different inputs
        wl = bench.rank_workload(W.TINY_BF16, rank)
        q, _, _, _ = W.make_inputs(wl)
        out[rank] = (mx, wl.seed, float(q.float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_replicas():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] != out[1][1]
    assert out[0][2] != out[1][2]


def test_reduce_max_without_group():
    import bench
    assert bench.reduce_max(3.5, None, torch.device("cpu")) == 3.5
