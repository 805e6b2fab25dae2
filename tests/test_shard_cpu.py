"""Sharding one layer across ranks (gloo, world size 2, CPU).

Kernels cannot run here, so each rank runs the oracle on its shard: the
test checks the partition (balanced, disjoint, complete), the shard views
(every unit sees exactly the data it sees unsharded) and the gather, against
the oracle's unsharded result, which the sharded one must equal exactly.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_kv_b200 import shard, synth


def _layer():
    w = synth.custom("shard_cpu", 5, 12, 3, [700, 33, 1500, 0, 260], [16, 32, 64], 128,
                     seed=21)
    return synth.make_layer(w, 0, "cpu")


def _oracle_out(d):
    from oracle import absp_oracle as O
    return O.run_layer(synth.host_layer(d)).out


def test_plans_are_balanced_disjoint_and_complete():
    lens = [700, 33, 1500, 0, 260, 4097, 16]
    for world in (1, 2, 3, 8):
        parts = shard.plan_by_sequence(lens, world)
        flat = sorted(s for p in parts for s in p)
        assert flat == list(range(len(lens)))
        assert all(p == sorted(p) for p in parts)
        loads = [sum(lens[s] for s in p) for p in parts]
        assert max(loads) - min(loads) <= max(lens)      # LPT bound
    assert shard.plan_by_sequence([5, 9, 7], 2) == [[1], [0, 2]]
    assert shard.plan_by_kv_head(8, 3) == [range(0, 3), range(3, 6), range(6, 8)]
    assert shard.plan_by_kv_head(2, 4) == [range(0, 1), range(1, 2), range(2, 2),
                                           range(2, 2)]


def test_shards_reassemble_to_the_unsharded_oracle_in_one_process():
    d = _layer()
    full = _oracle_out(d)
    G = d.num_q_heads // d.num_kv_heads
    for axis, plan in (("seq", shard.plan_by_sequence(d.seq_lens.tolist(), 2)),
                       ("kv_head", shard.plan_by_kv_head(d.num_kv_heads, 2))):
        parts = []
        for sh in plan:
            sd = shard.shard_sequences(d, sh) if axis == "seq" else shard.shard_kv_heads(d, sh)
            parts.append(None if sd is None else _oracle_out(sd))
        got = shard.assemble(parts, plan, axis, d.num_seqs, d.num_q_heads, G)
        assert np.array_equal(got, full), axis


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, axis, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = _layer()                       # every rank generates the same layer
        G = d.num_q_heads // d.num_kv_heads
        if axis == "seq":
            plan = shard.plan_by_sequence(d.seq_lens.tolist(), world)
            sd = shard.shard_sequences(d, plan[rank])
        else:
            plan = shard.plan_by_kv_head(d.num_kv_heads, world)
            sd = shard.shard_kv_heads(d, plan[rank])
        local = None if sd is None else _oracle_out(sd)
        full = shard.all_gather_outputs(local, plan, axis, d.num_seqs, d.num_q_heads, G, dist)
        q.put((rank, axis, full))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("axis", ["seq", "kv_head"])
def test_two_ranks_gather_the_unsharded_result(axis):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, axis, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = _oracle_out(_layer())
    for rank, ax, full in out:
        assert ax == axis
        assert np.array_equal(full, want), (rank, axis)
