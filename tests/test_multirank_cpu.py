"""Host logic of the multi-GPU path on CPU: world_size-2 gloo ranks.

The hot path has no exchange step: each rank runs an independent replica (weak scaling) or a
block of independent (batch, kv-head) units.  These tests cover the unit partition and the
max-over-ranks timing reduction bench.py uses."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, n_units, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = list(W.shard_units(n_units, rank, world))
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        t = bench.max_over_ranks(float(rank + 1) * 1.5, world)
        q.put((rank, gathered, t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_units", [1, 7, 32])
def test_units_partition_and_max_timing(n_units):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n_units, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gathered, t in res:
        flat = [u for part in gathered for u in part]
        assert sorted(flat) == list(range(n_units))  # every unit exactly once
        assert t == 3.0  # max over ranks of (rank + 1) * 1.5


def test_shard_units_balanced():
    for n in range(0, 50):
        for world in (1, 2, 3, 8):
            sizes = [len(W.shard_units(n, r, world)) for r in range(world)]
            assert sum(sizes) == n and max(sizes) - min(sizes) <= 1
