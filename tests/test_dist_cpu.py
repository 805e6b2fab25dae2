"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The decode path shards with no exchange: each rank decodes its own layer
stack, and the only collectives are the barrier and the max-over-ranks
reduction of the timed region.
"""

import datetime
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


class _FakeSampler:
    """Hands out prepared clock records, one per timed region."""

    def __init__(self, records):
        self.records = records

    def start(self):
        pass

    def stop(self):
        return self.records.pop(0)


def _remeasure_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    # a short timeout: ranks that took different collective steps end with
    # an error instead of waiting
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}
        slow = {**ok, "reasons": ["hw_slowdown"]}
        # only rank 1's first region saw a slowdown
        records = [dict(slow) if rank == 1 else dict(ok), dict(ok)]
        calls = []

        def timed():
            calls.append(1)
            dist.barrier()                          # a collective, as the real region has
            return bench.reduce_max(10.0 * len(calls) + rank, dist, "cpu")

        ms, clocks = bench.timed_with_clocks(timed, lambda: _FakeSampler(records), dist, "cpu")
        q.put((rank, len(calls), ms, clocks))
    finally:
        dist.destroy_process_group()


def test_slowdown_on_one_rank_retimes_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_remeasure_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ncalls, ms, clocks in out:
        assert ncalls == 2                          # both ranks timed again
        assert ms == 21.0                           # the second region, max over ranks
        assert clocks["reasons"] == []
        first = clocks["remeasured_after"]
        assert first["ms"] == 11.0
        assert first["why"] == (["hw_slowdown"] if rank == 1 else [])


def test_clean_clocks_time_once():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}
    calls = []

    def timed():
        calls.append(1)
        return 5.0

    ms, clocks = bench.timed_with_clocks(timed, lambda: _FakeSampler([dict(ok)]))
    assert (ms, len(calls)) == (5.0, 1) and "remeasured_after" not in clocks
