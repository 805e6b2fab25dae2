"""Seeded generator: determinism, shapes and the planted structure."""

import numpy as np
import torch

from block_sparse_attention_kv_b200 import synth


def test_layer_is_deterministic_on_cpu():
    w = synth.custom("det", 2, 8, 2, [300, 129], [16, 64], 128, seed=7)
    a = synth.make_layer(w, 0, "cpu")
    b = synth.make_layer(w, 0, "cpu")
    for x, y in ((a.q, b.q), (a.k_pages, b.k_pages), (a.v_pages, b.v_pages)):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    assert torch.equal(a.page_table, b.page_table)


def test_page_table_is_permutation_and_tails_are_nan():
    w = synth.custom("pt", 3, 4, 1, [33, 16, 70], [32], 64, seed=2)
    d = synth.make_layer(w, 0, "cpu")
    pt = d.page_table.numpy()
    used = np.concatenate([pt[0, :3], pt[1, :1], pt[2, :5]])
    assert sorted(used.tolist()) == list(range(9))
    assert np.all(pt[1, 1:] == -1)
    # sequence 0 has 33 tokens: slots 1..15 of its third page are NaN
    last = d.k_pages[pt[0, 2], 0].float()
    assert torch.isfinite(last[0]).all() and torch.isnan(last[1:]).all()


def test_block_size_mix_and_named_shapes():
    w = synth.WORKLOADS["llama31_8b_32k"]
    counts = {16: 0, 32: 0, 64: 0}
    for layer in range(400):
        for b in synth.draw_block_sizes(w, layer):
            counts[int(b)] += 1
    tot = sum(counts.values())
    assert abs(counts[64] / tot - 0.5) < 0.03
    assert abs(counts[16] / tot - 0.25) < 0.03
    p = synth.plan_layer(w, 0)
    assert p.max_pages == 32768 // 16 and p.num_phys_pages == 2048
    assert synth.WORKLOADS["tiny_8k"].block_sizes == (16, 64)
    g = synth.plan_layer(synth.WORKLOADS["gqa16_batch96_16k"], 0)
    assert g.seq_lens.shape == (96,) and np.all(g.seq_lens == 16384)
    assert g.block_size.tolist() == [16, 64]
    assert synth.WORKLOADS["gqa16_batch96_16k"].num_q_heads // 2 == 16


def test_ragged_lengths_log_uniform_range():
    w = synth.WORKLOADS["ragged64_paged"]
    lens = synth.draw_seq_lens(w)
    assert lens.shape == (64,)
    assert lens.min() >= 4096 and lens.max() <= 65536
    assert np.any(lens % 16 != 0)        # ragged page tails occur


def test_planted_spans_inside_sequence():
    w = synth.custom("pl", 1, 4, 2, [1000], [16, 32], 256, seed=3)
    p = synth.plan_layer(w, 0)
    for h in range(2):
        st = p.planted[0][h]
        assert len(st) == 8 and np.all(st % 64 == 0) and np.all(st + 64 <= 1000)
