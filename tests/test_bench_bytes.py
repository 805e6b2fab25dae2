"""The roofline numerator: algorithmic bytes of one decode layer-step.

bench.step_bytes counts, per (sequence, KV head), the centroid code rows
(64 B each), the per-channel scale and zero point (128 x 8 B), and 512 B
(one K row and one V row of 128 bf16) per valid selected token; plus the
query read and the output written (S x Hq x 256 B each).  Here it is checked
against a hand count and against the oracle's own selection, independently
of the CUDA path.
"""

import numpy as np

import bench
from block_sparse_attention_kv_b200 import synth
from oracle import absp_oracle as O


def _sel_arrays(res, S, Hkv):
    kmax = max(len(r.sel) for r in res.heads.values())
    sel = np.full((S, Hkv, max(kmax, 1)), -1, dtype=np.int64)
    cnt = np.zeros((S, Hkv), dtype=np.int64)
    for (s, h), r in res.heads.items():
        sel[s, h, :len(r.sel)] = r.sel
        cnt[s, h] = len(r.sel)
    return sel, cnt


def test_hand_count_with_ragged_last_block():
    # one sequence of 100 tokens, one KV head of block size 32, two query
    # heads: 4 code rows; blocks 0 and 3 hold 32 + 4 valid tokens
    w = synth.custom("bytes", 1, 2, 1, [100], [32], 64, seed=5)
    d = synth.make_layer(w, 0, "cpu")
    sel = np.array([[[0, 3]]])
    cnt = np.array([[2]])
    expect = 4 * 64 + 128 * 8 + 36 * 512 + 1 * 2 * 256 * 2
    assert bench.step_bytes(d, sel, cnt) == expect


def test_bf16_centroids_and_block_size_override():
    w = synth.custom("bytes", 1, 2, 1, [100], [32], 64, seed=5)
    d = synth.make_layer(w, 0, "cpu")
    # block size 16 instead: 7 rows of 256 B (bf16) and no INT4 parameters;
    # block 6 holds tokens 96..99
    sel = np.array([[[1, 6]]])
    cnt = np.array([[2]])
    expect = 7 * 256 + 20 * 512 + 2 * 256 * 2
    assert bench.step_bytes(d, sel, cnt, block_size=[16], bf16=True) == expect


def _independent_count(hl, res, Hq):
    total = hl.q_bits.shape[0] * Hq * 256 * 2
    for (s, h), r in res.heads.items():
        L, bs = int(hl.seq_lens[s]), int(hl.block_size[h])
        total += O.num_blocks(L, bs) * 64 + 128 * 8
        total += len(O.selected_tokens(r.sel, bs, L)) * 512
    return total


def test_matches_oracle_selection_on_ragged_layer():
    w = synth.custom("bytes", 3, 8, 2, [700, 1234, 0], [16, 64], 256, seed=11)
    d = synth.make_layer(w, 0, "cpu")
    hl = synth.host_layer(d)
    res = O.run_layer(hl)
    sel, cnt = _sel_arrays(res, 3, 2)
    assert bench.step_bytes(d, sel, cnt) == _independent_count(hl, res, 8)


def _full_length_closed_form(w, layer):
    # every sequence spans the whole context, so each head reads exactly
    # floor(budget / bs) * bs = budget tokens (the budget is a multiple of 64)
    bs = synth.draw_block_sizes(w, layer)
    per_seq = sum(w.ctx // int(b) * 64 + 128 * 8 + w.budget * 512 for b in bs)
    return w.num_seqs * (per_seq + w.num_q_heads * 256 * 2)


def test_llama31_8b_32k_layer0_from_oracle_selection():
    w = synth.WORKLOADS["llama31_8b_32k"]
    d = synth.make_layer(w, 0, "cpu")
    hl = synth.host_layer(d)
    res = O.run_layer(hl)
    sel, cnt = _sel_arrays(res, 1, 8)
    n = bench.step_bytes(d, sel, cnt)
    assert n == _independent_count(hl, res, 32)
    assert n == _full_length_closed_form(w, 0)


def test_llama31_8b_32k_mean_over_the_benchmarks_64_layers():
    # bytes_per_launch in the benchmark line is the mean over its 64 layer
    # caches (layer seeds 0..63 on rank 0), each with its own block sizes
    w = synth.WORKLOADS["llama31_8b_32k"]
    mean = np.mean([_full_length_closed_form(w, l) for l in bench.rank_layer_ids(0, 64)])
    assert mean == 8_935_424


def test_oracle_sample_lengths_span_a_ragged_batch():
    lens = np.arange(1, 65) * 1000
    assert bench.sample_lengths(lens, 4) == [9000, 25000, 41000, 57000]
    assert bench.sample_lengths([5, 3], 4) == [3, 5]
    w = synth.WORKLOADS["ragged64_paged"]
    pick = bench.sample_lengths(synth.draw_seq_lens(w), 4)
    assert pick == sorted(pick) and set(pick) <= set(synth.draw_seq_lens(w).tolist())


def test_oracle_workload_sample_keeps_the_workload_shape():
    prep, G, budget, pick, units = bench.oracle_workload_sample("gqa16_batch96_16k", k=2)
    w = synth.WORKLOADS["gqa16_batch96_16k"]
    assert G == 16 and budget == w.budget and units == 96 * 2
    assert pick == [16384, 16384] and len(prep) == 2 * 2
    assert sorted({u[5] for u in prep}) == [16, 64]          # the per-head block sizes
