"""The N > 1 host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

Each rank gets an independent, differently seeded shard (the method has no
exchange step), the timing reduction returns the slowest rank's time on every
rank, and the whole-job rate counts every rank's units over that time.
"""
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
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        w, r, local = bench.dist_setup()
        p, d = bench.shard_specs(r)
        t = bench.reduce_max(10.0 + 5.0 * r, w, "cpu")
        bench.barrier(w)
        out[rank] = (w, r, local, p.seed, d.seed, t,
                     bench.weak_scaling_rate(3.0, 2, w, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    r0, r1 = out[0], out[1]
    assert r0[:3] == (2, 0, 0) and r1[:3] == (2, 1, 1)
    assert r0[3] != r1[3] and r0[4] != r1[4]          # independent shards
    assert r0[5] == r1[5] == 15.0                      # max over ranks, on every rank
    assert r0[6] == pytest.approx(2 * 3.0 * 2 / 15e-3)  # all ranks' units / slowest time


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.reduce_max(4.0, 1, "cpu") == 4.0
    bench.barrier(1)
