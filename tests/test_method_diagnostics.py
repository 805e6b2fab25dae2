"""Method diagnostics on the synthetic inputs (oracle only, CPU).

The page's Fig. 8 reports top-K page recall above 0.9 in every layer for
INT4 asymmetric per-channel centroids (against full-precision ones); on the
seeded Llama-3.1-8B-shaped layer the same measure, averaged over the KV
heads, is checked to clear 0.9 too, with BF16 centroids closer still.
"""

import numpy as np

from block_sparse_attention_kv_b200 import synth
from oracle import diagnostics as D


def test_recall_definitions_by_hand():
    assert D.page_recall([1, 4, 7], [4, 7, 9, 12]) == 0.5
    assert D.page_recall([], []) == 1.0
    # a budget that covers the whole sequence recalls every token
    w = synth.custom("diag", 1, 4, 1, [200], [32], 4096, seed=4)
    hl = synth.host_layer(synth.make_layer(w, 0, "cpu"))
    assert D.token_recall(hl, 0, 0, np.arange(7), 32) == 1.0
    # no block selected: nothing recalled
    assert D.token_recall(hl, 0, 0, np.zeros(0, dtype=np.int64), 32) == 0.0


def test_int4_page_recall_on_the_llama_shaped_layer():
    w = synth.WORKLOADS["llama31_8b_32k"]
    hl = synth.host_layer(synth.make_layer(w, 0, "cpu"))
    d = D.layer_diagnostics(hl)
    int4 = np.mean([v["int4_page_recall"] for v in d.values()])
    bf16 = np.mean([v["bf16_page_recall"] for v in d.values()])
    assert int4 > 0.9                      # Fig. 8's bar, on synthetic keys
    assert bf16 >= int4
    assert all(v["int4_page_recall"] > 0.8 for v in d.values())


def test_planted_spans_are_recalled_on_configs_0_to_2():
    for name, layer in (("tiny_8k", 0), ("llama31_8b_32k", 0), ("qwen3_8b_128k_36l", 35)):
        d = synth.make_layer(synth.WORKLOADS[name], layer, "cpu")
        hl = synth.host_layer(d)
        assert D.planted_recall(hl, lambda s, h: synth.planted_mask(d.plan, s, h)) == 1.0, name
