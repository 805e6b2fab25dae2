"""Seeded synthetic decode workloads (inputs only).

This module builds the inputs that both the CUDA path and the CPU oracle
consume: a paged bf16 K/V cache for one attention layer, a page table, the
sequence lengths, the decode queries and the per-KV-head block-size table.
It holds none of the method's arithmetic (no centroids, quantisation,
scores, selection or attention).

Shapes follow the model shapes named for AB-Sparse (arXiv 2605.12110):
Llama-3.1-8B / Qwen3-8B attention (32 query heads, 8 KV heads, head_dim 128),
block sizes {16, 32, 64} per KV head (Fig. 3 / Fig. 5), a paged cache of
16-token physical pages with logical blocks mapped over them (Fig. 9).

Value recipe (per layer):
  * q ~ N(0, 1), rounded to bf16.
  * K ~ N(0, 1) plus +6 on 4 seeded channels per KV head (key-channel
    outliers, Fig. 7 shows centroid channels with large offsets), plus 8
    planted 64-token spans per (sequence, KV head) whose keys get
    +2 * qbar/|qbar| with qbar the sum of that head's GQA query group;
    rounded to bf16 once.
  * V ~ N(0, 1), rounded to bf16.
  * Physical page ids are a seeded random permutation.  Token slots past a
    sequence's length inside its last page are filled with NaN so that any
    consumer that reads them is caught.

Host-side choices (block sizes, lengths, outlier channels, planted spans,
page permutation) come from a numpy Generator, so they are identical on any
device; the bulk normal draws use a torch Generator on the target device.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional, Sequence

import numpy as np
import torch

HEAD_DIM = 128
PAGE_SIZE = 16
BLOCK_SIZES = (16, 32, 64)
BLOCK_SIZE_PROBS = (0.25, 0.25, 0.5)
BF16_NAN_BITS = 0x7FC0


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (shape + seeds)."""

    name: str
    layers: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    budget: int                      # token budget per KV head
    ctx: int = 0                     # fixed context length (0 when ragged)
    ragged: Optional[tuple] = None   # (lo, hi): lengths log-uniform in [lo, hi]
    block_sizes: Optional[tuple] = None  # fixed per-KV-head table, else drawn
    outlier_channels: int = 4
    outlier_bias: float = 6.0
    planted_blocks: int = 8
    planted_len: int = 64
    planted_gain: float = 2.0
    # per-KV-head span lengths (tokens): when given, head h gets
    # planted_tokens // planted_lens[h] spans of that length at arbitrary
    # token offsets (heads of different concentration); else the spans above
    planted_lens: Optional[tuple] = None
    planted_tokens: int = 512
    spare_pages: int = 0
    seed: int = 0


WORKLOADS = {
    # 1 layer, 2 KV heads with block sizes 16 and 64, GQA 4, 8K context.
    "tiny_8k": Workload("tiny_8k", layers=1, num_seqs=1, num_q_heads=8,
                        num_kv_heads=2, ctx=8192, budget=1024,
                        block_sizes=(16, 64), seed=1000),
    # Llama-3.1-8B-shaped attention layer, batch 1, 32K context.
    "llama31_8b_32k": Workload("llama31_8b_32k", layers=1, num_seqs=1,
                               num_q_heads=32, num_kv_heads=8, ctx=32768,
                               budget=2048, seed=1001),
    # Qwen3-8B-shaped decode step over 36 layers, 128K context.
    "qwen3_8b_128k_36l": Workload("qwen3_8b_128k_36l", layers=36, num_seqs=1,
                                  num_q_heads=32, num_kv_heads=8, ctx=131072,
                                  budget=4096, seed=1002),
    # Batched throughput: 32 sequences x 32K, 8 layers.
    "batch32_32k_8l": Workload("batch32_32k_8l", layers=8, num_seqs=32,
                               num_q_heads=32, num_kv_heads=8, ctx=32768,
                               budget=1024, seed=1003),
    # Ragged paged batch: 64 sequences, lengths log-uniform in [4096, 65536].
    "ragged64_paged": Workload("ragged64_paged", layers=1, num_seqs=64,
                               num_q_heads=32, num_kv_heads=8,
                               ragged=(4096, 65536), budget=2048, seed=1004),
    # GQA 16 batch: 96 sequences x 16K, 32 query heads over 2 KV heads
    # (block sizes 16 and 64), the widest group the kernels take.
    "gqa16_batch96_16k": Workload("gqa16_batch96_16k", layers=1, num_seqs=96,
                                  num_q_heads=32, num_kv_heads=2, ctx=16384,
                                  budget=1024, block_sizes=(16, 64), seed=1007),
    # Full centroid rebuild + INT4 quantisation at batch 8 x 131072.
    "rebuild_8x128k": Workload("rebuild_8x128k", layers=1, num_seqs=8,
                               num_q_heads=32, num_kv_heads=8, ctx=131072,
                               budget=2048, seed=1005),
    # Block-size sensitivity: 8 KV heads whose 512 relevant tokens come in
    # spans of 4 .. 512 tokens (concentrated to spread), 32K context.
    "calib_8h_32k": Workload("calib_8h_32k", layers=1, num_seqs=1,
                             num_q_heads=32, num_kv_heads=8, ctx=32768,
                             budget=2048, block_sizes=(16,) * 8,
                             planted_lens=(4, 8, 16, 32, 64, 128, 256, 512),
                             planted_tokens=512, seed=1006),
}


def custom(name: str, num_seqs: int, num_q_heads: int, num_kv_heads: int,
           seq_lens: Sequence[int], block_sizes: Sequence[int], budget: int,
           seed: int, **kw) -> "Workload":
    """A small workload with explicit lengths and block sizes (test cases)."""
    lens = tuple(int(x) for x in seq_lens)
    assert len(lens) == num_seqs
    return Workload(name, layers=1, num_seqs=num_seqs, num_q_heads=num_q_heads,
                    num_kv_heads=num_kv_heads, budget=budget,
                    ragged=("fixed",) + lens, block_sizes=tuple(block_sizes),
                    seed=seed, **kw)


@dataclass
class LayerPlan:
    """Host-side (device independent) choices for one layer."""

    workload: Workload
    layer: int
    seq_lens: np.ndarray            # int32 [S]
    block_size: np.ndarray          # int32 [Hkv]
    outlier_ch: np.ndarray          # int64 [Hkv][outlier_channels]
    planted: list                   # planted[s][h] -> array of span starts (tokens)
    page_table: np.ndarray          # int32 [S][max_pages], -1 where unused
    num_phys_pages: int
    max_pages: int


def _rng(w: Workload, layer: int, salt: int) -> np.random.Generator:
    return np.random.default_rng([int(w.seed), int(layer), int(salt)])


def draw_block_sizes(w: Workload, layer: int) -> np.ndarray:
    if w.block_sizes is not None:
        bs = np.asarray(w.block_sizes, dtype=np.int32)
        assert bs.shape == (w.num_kv_heads,)
        return bs
    r = _rng(w, layer, 1)
    return r.choice(np.asarray(BLOCK_SIZES), size=w.num_kv_heads,
                    p=np.asarray(BLOCK_SIZE_PROBS)).astype(np.int32)


def draw_seq_lens(w: Workload) -> np.ndarray:
    if w.ragged is None:
        return np.full(w.num_seqs, w.ctx, dtype=np.int32)
    if w.ragged[0] == "fixed":
        return np.asarray(w.ragged[1:], dtype=np.int32)
    lo, hi = w.ragged
    r = _rng(w, 0, 2)
    u = r.uniform(math.log(lo), math.log(hi), size=w.num_seqs)
    return np.clip(np.floor(np.exp(u)), lo, hi).astype(np.int32)


def planted_len(w: Workload, h: int) -> int:
    """Length of KV head h's planted spans (tokens)."""
    return int(w.planted_lens[h]) if w.planted_lens is not None else int(w.planted_len)


def planted_mask(plan: "LayerPlan", s: int, h: int) -> np.ndarray:
    """Token mask of the planted (q-aligned) keys of (sequence s, KV head h)."""
    L = int(plan.seq_lens[s])
    m = np.zeros(L, dtype=bool)
    ln = planted_len(plan.workload, h)
    for st in plan.planted[s][h]:
        m[int(st):min(L, int(st) + ln)] = True
    return m


def plan_layer(w: Workload, layer: int = 0) -> LayerPlan:
    S, Hkv = w.num_seqs, w.num_kv_heads
    lens = draw_seq_lens(w)
    bs = draw_block_sizes(w, layer)
    r = _rng(w, layer, 3)
    outl = np.stack([r.choice(HEAD_DIM, size=w.outlier_channels, replace=False)
                     for _ in range(Hkv)]).astype(np.int64) \
        if w.outlier_channels > 0 else np.zeros((Hkv, 0), np.int64)
    planted = []
    for s in range(S):
        row = []
        for h in range(Hkv):
            if w.planted_lens is None:
                nspan = int(lens[s]) // w.planted_len
                k = min(w.planted_blocks, nspan)
                starts = np.sort(r.choice(nspan, size=k, replace=False)) * w.planted_len \
                    if k > 0 else np.zeros(0, np.int64)
            else:
                # spans of length ln at any offset inside disjoint 2*ln slots
                ln = int(w.planted_lens[h])
                nslot = int(lens[s]) // (2 * ln)
                k = min(max(1, w.planted_tokens // ln), nslot)
                slots = np.sort(r.choice(nslot, size=k, replace=False)) if k > 0 \
                    else np.zeros(0, np.int64)
                starts = slots * (2 * ln) + r.integers(0, ln + 1, size=k)
            row.append(np.asarray(starts, dtype=np.int64))
        planted.append(row)
    pages_per_seq = [(int(L) + PAGE_SIZE - 1) // PAGE_SIZE for L in lens]
    max_pages = max(1, max(pages_per_seq))
    used = int(sum(pages_per_seq))
    num_phys = used + int(w.spare_pages)
    perm = _rng(w, layer, 4).permutation(max(num_phys, 1)).astype(np.int32)
    pt = np.full((S, max_pages), -1, dtype=np.int32)
    off = 0
    for s in range(S):
        n = pages_per_seq[s]
        pt[s, :n] = perm[off:off + n]
        off += n
    return LayerPlan(w, layer, lens, bs, outl, planted, pt, max(num_phys, 1),
                     max_pages)


@dataclass
class LayerData:
    """Device tensors for one layer (all torch, on one device)."""

    plan: LayerPlan
    q: torch.Tensor            # bf16 [S][Hq][128]
    k_pages: torch.Tensor      # bf16 [P][Hkv][16][128]
    v_pages: torch.Tensor      # bf16 [P][Hkv][16][128]
    page_table: torch.Tensor   # int32 [S][max_pages]
    seq_lens: torch.Tensor     # int32 [S]
    block_size: np.ndarray     # int32 [Hkv] (host)
    budget: int

    @property
    def num_seqs(self):
        return self.q.shape[0]

    @property
    def num_q_heads(self):
        return self.q.shape[1]

    @property
    def num_kv_heads(self):
        return self.k_pages.shape[1]


def _torch_gen(device, w: Workload, layer: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(w.seed) * 100003 + int(layer) * 7919 + 17)
    return g


def make_layer(w: Workload, layer: int = 0, device="cpu",
               plan: Optional[LayerPlan] = None,
               tail_fill_nan: bool = True) -> LayerData:
    """Generate one layer of `w` on `device` (deterministic per device)."""
    plan = plan or plan_layer(w, layer)
    dev = torch.device(device)
    S, Hq, Hkv, D = w.num_seqs, w.num_q_heads, w.num_kv_heads, HEAD_DIM
    G = Hq // Hkv
    g = _torch_gen(dev, w, layer)
    q = torch.randn((S, Hq, D), generator=g, device=dev,
                    dtype=torch.float32).to(torch.bfloat16)
    P = plan.num_phys_pages
    fill = float("nan") if tail_fill_nan else 0.0
    k_pages = torch.full((P, Hkv, PAGE_SIZE, D), fill, dtype=torch.bfloat16,
                         device=dev)
    v_pages = torch.full((P, Hkv, PAGE_SIZE, D), fill, dtype=torch.bfloat16,
                         device=dev)
    qbar = q.float().view(S, Hkv, G, D).sum(dim=2)            # [S][Hkv][D]
    u = qbar / qbar.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    outl = torch.as_tensor(plan.outlier_ch, device=dev)
    pt = torch.as_tensor(plan.page_table, device=dev)
    for s in range(S):
        L = int(plan.seq_lens[s])
        npg = (L + PAGE_SIZE - 1) // PAGE_SIZE
        if npg == 0:
            continue
        kk = torch.randn((L, Hkv, D), generator=g, device=dev,
                         dtype=torch.float32)
        if outl.shape[1] > 0:
            bias = torch.zeros((Hkv, D), device=dev, dtype=torch.float32)
            bias.scatter_(1, outl, w.outlier_bias)
            kk += bias
        for h in range(Hkv):
            ln = planted_len(w, h)
            for st in plan.planted[s][h]:
                st = int(st)
                kk[st:st + ln, h, :] += w.planted_gain * u[s, h]
        vv = torch.randn((L, Hkv, D), generator=g, device=dev,
                         dtype=torch.float32)
        pad = npg * PAGE_SIZE - L
        kb = kk.to(torch.bfloat16)
        vb = vv.to(torch.bfloat16)
        if pad:
            tail = torch.full((pad, Hkv, D), fill, dtype=torch.bfloat16,
                              device=dev)
            kb = torch.cat([kb, tail])
            vb = torch.cat([vb, tail])
        ids = pt[s, :npg].long()
        k_pages[ids] = kb.view(npg, PAGE_SIZE, Hkv, D).permute(0, 2, 1, 3)
        v_pages[ids] = vb.view(npg, PAGE_SIZE, Hkv, D).permute(0, 2, 1, 3)
        del kk, vv, kb, vb
    return LayerData(plan, q, k_pages, v_pages, pt.to(torch.int32),
                     torch.as_tensor(plan.seq_lens, device=dev),
                     plan.block_size.copy(), int(w.budget))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a host uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@dataclass
class HostLayer:
    """Host (numpy) copy of the part of a layer that some sequences touch."""

    seqs: list                 # original sequence ids, in order
    q_bits: np.ndarray         # uint16 [S'][Hq][128]
    k_bits: np.ndarray         # uint16 [P'][Hkv][16][128]
    v_bits: np.ndarray         # uint16 [P'][Hkv][16][128]
    page_table: np.ndarray     # int32 [S'][max_pages] (renumbered pages)
    seq_lens: np.ndarray       # int32 [S']
    block_size: np.ndarray     # int32 [Hkv]
    budget: int


def host_layer(d: LayerData, seqs: Optional[Sequence[int]] = None) -> HostLayer:
    """Copy the pages, page-table rows and queries of `seqs` to the host.

    Pages are renumbered densely; the page table is remapped accordingly,
    so the copy is a self-contained paged layer of len(seqs) sequences.
    """
    seqs = list(range(d.num_seqs)) if seqs is None else [int(s) for s in seqs]
    pt_all = d.page_table.cpu().numpy()
    lens_all = d.seq_lens.cpu().numpy()
    pages = []
    rows = []
    for s in seqs:
        npg = (int(lens_all[s]) + PAGE_SIZE - 1) // PAGE_SIZE
        row = np.full(pt_all.shape[1], -1, dtype=np.int32)
        ids = pt_all[s, :npg]
        row[:npg] = np.arange(len(pages), len(pages) + npg, dtype=np.int32)
        pages.extend(int(x) for x in ids)
        rows.append(row)
    idx = torch.as_tensor(np.asarray(pages, dtype=np.int64),
                          device=d.k_pages.device)
    k = bf16_bits(d.k_pages.index_select(0, idx)) if len(pages) else \
        np.zeros((0,) + tuple(d.k_pages.shape[1:]), np.uint16)
    v = bf16_bits(d.v_pages.index_select(0, idx)) if len(pages) else \
        np.zeros((0,) + tuple(d.v_pages.shape[1:]), np.uint16)
    sidx = torch.as_tensor(seqs, device=d.q.device, dtype=torch.long)
    return HostLayer(seqs, bf16_bits(d.q.index_select(0, sidx)), k, v,
                     np.stack(rows).astype(np.int32),
                     lens_all[seqs].astype(np.int32), d.block_size.copy(),
                     d.budget)


def with_budget(w: Workload, budget: int) -> Workload:
    return replace(w, budget=int(budget))
