"""One layer's decode split across ranks (host logic: partition and gather).

Every (sequence, KV head) unit of steps 1-5 is independent of every other:
its centroids, per-channel INT4 parameters, scores, top-K and attention read
only that sequence's keys and values of that KV head and the queries of its
GQA group (AB-Sparse, arXiv 2605.12110, Fig. 1: each head scores and selects
its own blocks).  A layer therefore shards with no exchange inside the
attention, in either of two ways:

* by sequence: each rank decodes a subset of the batch and holds only the
  physical pages of its sequences;
* by KV head: each rank holds some KV heads' cache together with the whole
  query group of each of them (query head j belongs to KV head j // G).

Each rank runs the unchanged C-ABI calls on its shard; the only collective
is the gather of the outputs ([S][Hq][128]) after the step.  This module
holds the partition, the shard views and the reassembly; it does none of the
method's arithmetic.
"""

from __future__ import annotations

from dataclasses import replace
from typing import List, Sequence

import numpy as np
import torch

PAGE_SIZE = 16


def plan_by_sequence(seq_lens: Sequence[int], world: int) -> List[List[int]]:
    """Sequences per rank, balanced by tokens: longest first, each onto the
    rank with the fewest tokens so far (ties to the lower rank); every
    rank's list in ascending sequence order.  A rank may get none."""
    if world < 1:
        raise ValueError("world must be >= 1")
    lens = [int(x) for x in seq_lens]
    order = sorted(range(len(lens)), key=lambda s: (-lens[s], s))
    load = [0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for s in order:
        r = min(range(world), key=lambda i: (load[i], i))
        parts[r].append(s)
        load[r] += lens[s]
    return [sorted(p) for p in parts]


def plan_by_kv_head(num_kv_heads: int, world: int) -> List[range]:
    """Contiguous KV-head ranges per rank, sizes differing by at most one
    (the first num_kv_heads % world ranks get the extra head)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    base, extra = divmod(int(num_kv_heads), world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append(range(h, h + n))
        h += n
    return out


def shard_sequences(d, seqs: Sequence[int]):
    """The layer restricted to sequences `seqs`: their queries, lengths and
    page-table rows, and only their physical pages (renumbered densely in
    sequence order), which is what a rank holding them stores."""
    seqs = [int(s) for s in seqs]
    if not seqs:
        return None
    lens = d.seq_lens.cpu().numpy()
    pt = d.page_table.cpu().numpy()
    pages, rows = [], []
    for s in seqs:
        npg = (int(lens[s]) + PAGE_SIZE - 1) // PAGE_SIZE
        row = np.zeros(pt.shape[1], dtype=np.int32)
        row[:npg] = np.arange(len(pages), len(pages) + npg, dtype=np.int32)
        pages.extend(int(x) for x in pt[s, :npg])
        rows.append(row)
    dev = d.k_pages.device
    if pages:
        idx = torch.as_tensor(pages, dtype=torch.long, device=dev)
        k = d.k_pages.index_select(0, idx).contiguous()
        v = d.v_pages.index_select(0, idx).contiguous()
    else:   # only empty sequences: one unused page keeps the pool non-empty
        k = d.k_pages[:1].clone()
        v = d.v_pages[:1].clone()
    sidx = torch.as_tensor(seqs, dtype=torch.long, device=d.q.device)
    return replace(d, plan=None,
                   q=d.q.index_select(0, sidx).contiguous(),
                   k_pages=k, v_pages=v,
                   page_table=torch.as_tensor(np.stack(rows), device=dev),
                   seq_lens=d.seq_lens.index_select(0, sidx).contiguous(),
                   block_size=np.asarray(d.block_size).copy())


def shard_kv_heads(d, heads: range):
    """The layer restricted to KV heads `heads` with their whole query
    groups: K/V pages [P][len(heads)][16][128], queries [S][G*len(heads)][128]
    and those heads' block sizes (the page table and lengths are shared)."""
    if len(heads) == 0:
        return None
    G = d.num_q_heads // d.num_kv_heads
    h0, h1 = heads.start, heads.stop
    return replace(d, plan=None,
                   q=d.q[:, h0 * G:h1 * G].contiguous(),
                   k_pages=d.k_pages[:, h0:h1].contiguous(),
                   v_pages=d.v_pages[:, h0:h1].contiguous(),
                   block_size=np.asarray(d.block_size)[h0:h1].copy())


def assemble(parts, plan, axis: str, num_seqs: int, num_q_heads: int, group: int):
    """Full [S][Hq][128] output from the per-rank outputs `parts` (torch
    tensors or numpy arrays, None for a rank with an empty shard) of
    `plan` (from plan_by_sequence or plan_by_kv_head)."""
    first = next(p for p in parts if p is not None)
    if isinstance(first, torch.Tensor):
        out = torch.zeros((num_seqs, num_q_heads, first.shape[-1]), dtype=first.dtype,
                          device=first.device)
    else:
        out = np.zeros((num_seqs, num_q_heads, first.shape[-1]), dtype=first.dtype)
    for p, sh in zip(parts, plan):
        if p is None or len(sh) == 0:
            continue
        if axis == "seq":
            for i, s in enumerate(sh):
                out[s] = p[i]
        elif axis == "kv_head":
            out[:, sh.start * group:sh.stop * group] = p
        else:
            raise ValueError(f"unknown shard axis {axis!r}")
    return out


def all_gather_outputs(local, plan, axis: str, num_seqs: int, num_q_heads: int,
                       group: int, dist):
    """Every rank's output shard gathered into the full output on every rank
    (one all_gather of host objects; the shard sizes differ by rank)."""
    obj = None if local is None else (local.cpu().numpy() if isinstance(local, torch.Tensor)
                                      else np.asarray(local))
    parts = [None] * dist.get_world_size()
    dist.all_gather_object(parts, obj)
    return assemble(parts, plan, axis, num_seqs, num_q_heads, group)
