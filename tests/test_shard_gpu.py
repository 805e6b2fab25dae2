"""Sharding one layer across ranks on the GPU, one process standing in for
two ranks: each shard runs the unchanged C-ABI calls, the gathered output
and the per-unit selections match the unsharded run (selections exactly,
outputs within the parity tolerance: a shard may run with another cluster
size, which changes only the order of the softmax merge)."""

import pytest
import torch

from block_sparse_attention_kv_b200 import shard, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, pipeline
    return abi, pipeline


def _run(pipeline, d):
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    dl.score_select()
    dl.decode_step()
    dl.check()
    torch.cuda.synchronize()
    return dl


@pytest.mark.parametrize("wname,axis", [("llama31_8b_32k", "kv_head"),
                                        ("ragged_shard", "seq"),
                                        ("ragged_shard", "kv_head")])
def test_two_shards_match_the_unsharded_layer(lib, wname, axis):
    _, pipeline = lib
    w = synth.WORKLOADS.get(wname) or synth.custom(
        "ragged_shard", 6, 32, 8, [4097, 900, 33, 20000, 0, 1600],
        [16, 32, 64, 16, 64, 32, 16, 64], 1024, seed=31)
    d = synth.make_layer(w, 0, "cuda")
    full = _run(pipeline, d)
    G = d.num_q_heads // d.num_kv_heads
    if axis == "seq":
        plan = shard.plan_by_sequence(d.seq_lens.tolist(), 2)
    else:
        plan = shard.plan_by_kv_head(d.num_kv_heads, 2)
    outs = []
    for sh in plan:
        sd = shard.shard_sequences(d, sh) if axis == "seq" else shard.shard_kv_heads(d, sh)
        part = _run(pipeline, sd)
        outs.append(part.out)
        # the shard's selections are the unsharded ones of the same units
        if axis == "seq":
            for i, s in enumerate(sh):
                assert torch.equal(part.sel_count[i], full.sel_count[s])
                for h in range(d.num_kv_heads):
                    k = int(full.sel_count[s, h])
                    assert torch.equal(part.sel[i, h, :k], full.sel[s, h, :k])
        else:
            for i, h in enumerate(sh):
                assert torch.equal(part.sel_count[:, i], full.sel_count[:, h])
                k = int(full.sel_count[:, h].max())
                assert torch.equal(part.sel[:, i, :k], full.sel[:, h, :k])
    got = shard.assemble(outs, plan, axis, d.num_seqs, d.num_q_heads, G)
    diff = (got.float() - full.out.float()).abs()
    assert diff.max().item() <= 2e-2 and diff.mean().item() <= 2e-3
