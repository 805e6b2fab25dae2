"""Oracle for the per-head block-size sensitivity calibration.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).  It shares no code
with the library and imports nothing from it; the selections come from
`absp_oracle.run_layer`, the recall is counted token by token and the
allocation is found by trying every assignment.

What it computes (AB-Sparse, arXiv 2605.12110, head sensitivity analysis,
Fig. 3, and the rebuttal's accuracy-drop reading of it):

* for each candidate block size bs, every KV head of the layer is blocked
  at bs (same keys), centroids are built and INT4-quantised and the top-K
  blocks are selected exactly as in the decode path;
* the recall of a head at bs is the number of its relevant tokens that lie
  in a selected block, over the number of its relevant tokens, both summed
  over the sequences; normalised recall divides by the recall at the
  smallest candidate size (a head whose recall there is 0 gets 1);
* the allocation picks one block size per head so that the summed value
  (normalised recall) is largest with the centroid rows, sum over
  sequences of ceil(L / bs), within a row budget; ties go to the smaller
  total cost, then to the lexicographically smallest choice of option
  indices; values are summed in head order.

Reading (the pages leave open what "relevant" means): on synthetic layers
the relevant tokens are the planted keys aligned with the group's query,
the only tokens built to carry attention weight.
"""

from __future__ import annotations

import copy
import itertools

import numpy as np

from . import absp_oracle as O


def token_hits(sel_blocks, bs: int, length: int, relevant: np.ndarray) -> int:
    """Relevant tokens of [0, length) inside the blocks sel_blocks at size bs."""
    hits = 0
    chosen = set(int(b) for b in sel_blocks)
    for t in range(length):
        if relevant[t] and (t // bs) in chosen:
            hits += 1
    return hits


def calibrate(layer, relevant, block_sizes=(16, 32, 64)):
    """(hits [H][n], relevant totals [H], centroid rows [H][n]) of a host layer.

    relevant(s, h) -> bool array over the L_s tokens of (sequence s, head h).
    """
    S = len(layer.seq_lens)
    H = len(layer.block_size)
    n = len(block_sizes)
    hits = np.zeros((H, n), np.int64)
    rows = np.zeros((H, n), np.int64)
    rel = np.zeros(H, np.int64)
    for s in range(S):
        for h in range(H):
            rel[h] += int(np.count_nonzero(relevant(s, h)))
    for j, bs in enumerate(block_sizes):
        lay = copy.copy(layer)
        lay.block_size = np.full(H, bs, dtype=np.int32)
        res = O.run_layer(lay, with_attention=False)
        for h in range(H):
            for s in range(S):
                L = int(layer.seq_lens[s])
                rows[h, j] += -(-L // bs)
                hits[h, j] += token_hits(res.heads[(s, h)].sel, bs, L, relevant(s, h))
    return hits, rel, rows


def normalised_recall(hits, rel):
    hits = np.asarray(hits, dtype=np.float64)
    rel = np.asarray(rel, dtype=np.float64)
    out = np.ones_like(hits)
    for h in range(hits.shape[0]):
        if rel[h] == 0 or hits[h, 0] == 0:
            continue
        for j in range(hits.shape[1]):
            out[h, j] = (hits[h, j] / rel[h]) / (hits[h, 0] / rel[h])
    return out


def best_allocation(value, cost, budget):
    """Every assignment tried in lexicographic order: (choice, value, cost)."""
    value = np.asarray(value, dtype=np.float64)
    cost = np.asarray(cost, dtype=np.int64)
    H, n = value.shape
    best = None
    for ch in itertools.product(range(n), repeat=H):
        c = sum(int(cost[h, ch[h]]) for h in range(H))
        if c > budget:
            continue
        v = 0.0
        for h in range(H):
            v += float(value[h, ch[h]])
        if best is None or v > best[1] or (v == best[1] and c < best[2]):
            best = (tuple(ch), v, c)
    return best if best is not None else (None, -np.inf, 0)
