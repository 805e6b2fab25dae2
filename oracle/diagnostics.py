"""Method diagnostics on the synthetic inputs, computed with the oracle.

TEST INFRASTRUCTURE ONLY, like the rest of this package: nothing on the
product path imports it.  The CUDA path's selections equal the oracle's
(up to counted boundary near-ties), so these figures describe it too.

    python -m oracle.diagnostics [workload] [layers]

Per (sequence, KV head) of a layer:

* page recall of the INT4 selection: the share of the blocks selected with
  full-precision (fp64) centroids that the INT4-centroid selection also
  selects.  This is the synthetic analogue of the page's Fig. 8, which
  reports top-K page recall above 0.9 in every layer of Llama-3.1-8B for
  asymmetric per-channel INT4 centroids;
* the same for BF16 centroids (the page's Fig. 13 precision baseline);
* planted recall: the share of the planted q-aligned tokens inside the
  selected blocks (1.0 expected: they are what the generator makes
  relevant);
* token recall: the share of the exact top-budget tokens (by the group-summed
  query's dot product with each key) that lie in the selected blocks.  On
  i.i.d. synthetic keys a block mean cannot single out isolated tokens, so
  this stays low; the planted q-aligned spans are what the blocks capture.
"""

from __future__ import annotations

import sys

import numpy as np

from . import absp_oracle as O


def page_recall(sel, ref) -> float:
    """Share of the reference selection `ref` that `sel` also holds."""
    ref = set(int(b) for b in ref)
    return len(ref & set(int(b) for b in sel)) / len(ref) if ref else 1.0


def token_recall(layer, s: int, h: int, sel, bs: int) -> float:
    """Share of the top-budget tokens by qbar . k inside the blocks `sel`."""
    keys, _ = O.head_keys_values(layer, s, h)
    if keys.shape[0] == 0:
        return 1.0
    G = layer.q_bits.shape[1] // len(layer.block_size)
    qbar = O.group_query(O.decode_bf16(layer.q_bits[s]), h, G)
    dots = keys @ qbar
    B = min(int(layer.budget), dots.shape[0])
    top = np.lexsort((np.arange(dots.shape[0]), -dots))[:B]
    toks = set(O.selected_tokens(np.asarray(sel), bs, keys.shape[0]).tolist())
    return float(np.mean([int(t) in toks for t in top]))


def planted_recall(layer, planted_mask) -> float:
    """Share of the planted q-aligned tokens (planted_mask(s, h) -> bool mask
    over the sequence) inside the oracle's INT4 selection, over all
    (sequence, KV head) of the layer."""
    res = O.run_layer(layer, with_attention=False)
    hit = tot = 0
    for (s, h), hr in res.heads.items():
        m = np.asarray(planted_mask(s, h), dtype=bool)
        toks = O.selected_tokens(hr.sel, hr.block_size, hr.seq_len)
        tot += int(m.sum())
        hit += int(m[toks].sum())
    return hit / tot if tot else 1.0


def layer_diagnostics(layer) -> dict:
    """(s, h) -> {"int4_page_recall", "bf16_page_recall", "token_recall"}."""
    r4 = O.run_layer(layer, with_attention=False)
    rf = O.run_layer(layer, quantize=False, with_attention=False)
    rb = O.run_layer(layer, quantize="bf16", with_attention=False)
    out = {}
    for key, hr in sorted(r4.heads.items()):
        ref = rf.heads[key].sel
        out[key] = {"int4_page_recall": page_recall(hr.sel, ref),
                    "bf16_page_recall": page_recall(rb.heads[key].sel, ref),
                    "token_recall": token_recall(layer, key[0], key[1], hr.sel,
                                                 hr.block_size)}
    return out


def main(argv) -> None:
    from block_sparse_attention_kv_b200 import synth
    name = argv[1] if len(argv) > 1 else "llama31_8b_32k"
    layers = range(int(argv[2]) if len(argv) > 2 else 3)
    w = synth.WORKLOADS[name]
    for layer in layers:
        hl = synth.host_layer(synth.make_layer(w, layer, "cpu"))
        d = layer_diagnostics(hl)
        for (s, h), v in d.items():
            print(f"{name} layer {layer} seq {s} head {h} bs {int(hl.block_size[h])}: "
                  f"INT4 page recall {v['int4_page_recall']:.3f}, "
                  f"BF16 {v['bf16_page_recall']:.3f}, token recall {v['token_recall']:.3f}")
        means = {k: np.mean([v[k] for v in d.values()]) for k in next(iter(d.values()))}
        print(f"{name} layer {layer} mean: " +
              ", ".join(f"{k} {m:.3f}" for k, m in means.items()))


if __name__ == "__main__":
    main(sys.argv)
