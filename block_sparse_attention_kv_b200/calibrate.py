"""Per-KV-head block-size sensitivity calibration and block-size allocation.

AB-Sparse (arXiv 2605.12110), head sensitivity analysis, Fig. 3: attention
heads differ in how much they lose when key blocks grow; for some the
normalised recall of the relevant tokens stays flat from block size 16 to
64, for others it drops, which is why the block size is chosen per KV head.  This module measures that curve on a paged
layer and turns it into a block-size table:

1. for every block size in {16, 32, 64}, the whole layer is re-blocked at
   that size (same K/V cache, uniform table), centroids are built and
   quantised and the per-head top-K is selected, all by the library's own
   kernels (`DeviceLayer`);
2. recall of a head = the share of its relevant tokens that fall inside its
   selected blocks, summed over the sequences; the relevant tokens are given
   by the caller (on synthetic layers, the planted q-aligned keys);
3. normalised recall = recall(bs) / recall(16);
4. allocation: the block size of each head that maximises the summed
   normalised recall with the centroid store (rows of 64 bytes; a head at
   block size bs holds ceil(L / bs) rows per sequence) within a row budget,
   solved exactly by dynamic programming over heads.

Steps 2-4 are host bookkeeping on a few integers per head.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Sequence

import numpy as np
import torch

from .pipeline import DeviceLayer

BLOCK_SIZES = (16, 32, 64)


@dataclass
class Calibration:
    block_sizes: tuple          # the candidate block sizes, ascending
    hits: np.ndarray            # int64 [Hkv][nbs]: relevant tokens selected
    relevant: np.ndarray        # int64 [Hkv]: relevant tokens in total
    rows: np.ndarray            # int64 [Hkv][nbs]: centroid rows (all sequences)

    @property
    def recall(self) -> np.ndarray:
        """float64 [Hkv][nbs]: hits / relevant (0 where a head has none)."""
        rel = np.maximum(self.relevant, 1)[:, None]
        return np.where(self.relevant[:, None] > 0, self.hits / rel, 0.0)

    @property
    def normalised(self) -> np.ndarray:
        """Recall relative to the smallest block size (1 where that is 0)."""
        r = self.recall
        base = r[:, :1]
        return np.where(base > 0, r / np.where(base > 0, base, 1.0), 1.0)


def selected_token_mask(sel: np.ndarray, count: int, bs: int, length: int) -> np.ndarray:
    """Token mask of the blocks sel[:count] at block size bs (length tokens)."""
    m = np.zeros(length, dtype=bool)
    for b in np.asarray(sel[:count], dtype=np.int64):
        m[b * bs:min(length, (b + 1) * bs)] = True
    return m


def centroid_rows(seq_lens: Sequence[int], bs: int) -> int:
    return int(sum((int(L) + bs - 1) // bs for L in seq_lens))


def calibrate(data, relevant: Callable[[int, int], np.ndarray], budget: int = None,
              block_sizes: Sequence[int] = BLOCK_SIZES, stream=None) -> Calibration:
    """Selections of `data` (a device layer) at each uniform block size.

    relevant(s, h) -> bool mask over the L_s tokens of (sequence s, KV head h).
    """
    S, Hkv = data.num_seqs, data.num_kv_heads
    lens = [int(x) for x in data.seq_lens.cpu().tolist()]
    bss = tuple(int(b) for b in block_sizes)
    masks = [[np.asarray(relevant(s, h), dtype=bool) for h in range(Hkv)] for s in range(S)]
    hits = np.zeros((Hkv, len(bss)), np.int64)
    rows = np.zeros((Hkv, len(bss)), np.int64)
    rel = np.array([sum(int(masks[s][h].sum()) for s in range(S)) for h in range(Hkv)],
                   np.int64)
    for j, bs in enumerate(bss):
        dl = DeviceLayer(data, budget, stream, block_size=[bs] * Hkv)
        dl.build_centroids()
        dl.score_select()
        dl.check()
        if stream is not None:
            torch.cuda.current_stream().wait_stream(torch.cuda.ExternalStream(stream))
        sel = dl.sel.cpu().numpy()
        cnt = dl.sel_count.cpu().numpy()
        for h in range(Hkv):
            rows[h, j] = centroid_rows(lens, bs)
            for s in range(S):
                sm = selected_token_mask(sel[s, h], int(cnt[s, h]), bs, lens[s])
                hits[h, j] += int(np.count_nonzero(sm & masks[s][h]))
        del dl
    return Calibration(bss, hits, rel, rows)


def allocate(value: np.ndarray, cost: np.ndarray, budget: int):
    """Choose one option per head maximising the summed value within budget.

    value: float [H][n]; cost: integer [H][n] (e.g. centroid rows).  Returns
    (choice: tuple of H option indices, total value, total cost), or
    (None, -inf, 0) when even the cheapest choice exceeds the budget.  The
    optimum is taken as: largest value, then smallest cost, then the
    lexicographically smallest choice; values are summed in head order.
    Exact: dynamic programming over the heads on the Pareto frontier of
    (cost, value) states (a state is dropped when another costs no more and
    is worth at least as much, which never drops the optimum under this
    order).
    """
    value = np.asarray(value, dtype=np.float64)
    cost = np.asarray(cost, dtype=np.int64)
    H, n = value.shape
    states = [(0, 0.0, ())]
    for h in range(H):
        grown = []
        for c, v, ch in states:
            for j in range(n):
                cc = c + int(cost[h, j])
                if cc <= budget:
                    grown.append((cc, v + float(value[h, j]), ch + (j,)))
        grown.sort(key=lambda t: (t[0], -t[1], t[2]))
        states, best_v = [], -np.inf
        for t in grown:
            if t[1] > best_v:
                states.append(t)
                best_v = t[1]
        if not states:
            return None, -np.inf, 0
    c, v, ch = states[-1]   # costs ascend and values strictly ascend
    return ch, v, c
