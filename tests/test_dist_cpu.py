"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The decode path shards with no exchange: each rank decodes its own layer
stack, and the only collectives are the barrier and the max-over-ranks
reduction of the timed region.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]                     # rank 1 is the slower one
        mx = bench.reduce_max(ms, dist, "cpu")
        dist.barrier()
        ids = bench.rank_layer_ids(rank, 4)
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        q.put((rank, mx, gathered))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_max_and_disjoint_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered in out:
        assert mx == 20.0
        a, b = gathered
        assert set(a).isdisjoint(b) and len(a) == len(b) == 4


def test_single_process_rate_and_reduce():
    assert bench.reduce_max(3.5) == 3.5
    # 2 ranks x 64 layers x 100 steps in 200 ms
    assert bench.aggregate_rate(2, 64, 100, 200.0) == pytest.approx(64000.0)
    assert bench.rank_layer_ids(1, 3) == [3, 4, 5]
