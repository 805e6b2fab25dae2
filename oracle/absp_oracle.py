"""CPU oracle for adaptive-block sparse decode attention (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, the smoke check in ``__graft_entry__`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA
library and imports nothing from it.

What it computes follows AB-Sparse: Sparse Attention with Adaptive Block
Size (arXiv 2605.12110), as summarised on its review page:

* Fig. 1 (block-sparse paradigm): each key block is represented by a
  centroid; a query-centroid dot product gives each block an importance
  score; the top-K blocks are selected; attention runs over the keys of the
  selected blocks only.
* Fig. 3 / Fig. 5 / abstract: each KV head has its own block size, drawn
  from {16, 32, 64}, fixed offline; centroids are built once over all keys
  of a head.
* Fig. 8 / abstract: centroids are stored as INT4 codes, asymmetric
  quantisation with per-channel parameters.
* Fig. 9 (mapping strategy): logical blocks of a head are runs of ``bs/16``
  consecutive 16-token physical pages; heads with different block sizes
  select different numbers of blocks covering the same number of pages
  (TopK=1 at stride 4 vs TopK=2 at stride 2).

Where the pages leave a step open the oracle takes these readings:

* centroid = arithmetic mean of the block's valid keys (a ragged last block
  averages only its valid tokens); sums run in token order in fp64;
* per-channel statistics = min / max over all centroids of one
  (sequence, KV head); scale = fp32((max - min) / 15); zero point =
  rint(-min / scale) kept as an int32 (not clamped to 4 bits, saturated to
  the int32 range); code = clamp(rint(c / scale) + zp, 0, 15); rint is
  IEEE round-half-to-even; a channel with max == min (or a scale that
  rounds to 0 in fp32) gets scale 0, zp 0 and all codes 0;
* a GQA group's queries are summed into one vector qbar per KV head and
  the block score is qbar . dequant(code); the 1/sqrt(d) factor is left
  out (it does not change the ranking);
* the budget is in tokens: a head of block size bs keeps
  K = max(1, floor(budget / bs)) blocks (all blocks when it has fewer);
  ranking is by score descending, ties broken by the lower block index;
* no forced sink or local-window blocks;
* attention is exact softmax attention of each query head over the valid
  tokens of its KV head's selected blocks, logits q . k / sqrt(128).

Every step is written as plainly as possible; nothing is blocked, fused or
reordered.  Floating point is fp64 throughout (bf16 inputs convert
exactly); the only fp32 value is the stored scale, as specified above.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128
PAGE_SIZE = 16
CODE_LEVELS = 15          # INT4 asymmetric: codes 0..15


# ---------------------------------------------------------------- inputs --

def decode_bf16(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly.

    A bf16 number is the upper half of an IEEE binary32; widening the bit
    pattern by 16 zero bits gives that binary32, which fp64 holds exactly.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def gather_head_tokens(pages_bits, page_table_row, seq_len, kv_head):
    """Logical token rows [seq_len][128] (fp64) of one head from a paged cache.

    Token t lives in logical page t // 16 at slot t % 16; the page table maps
    the logical page to a physical page (Fig. 9, physical pages vs logical
    blocks).  Pages are laid out [page][kv_head][slot][channel].
    """
    t = np.arange(int(seq_len))
    phys = np.asarray(page_table_row, dtype=np.int64)[t // PAGE_SIZE]
    return decode_bf16(pages_bits[phys, kv_head, t % PAGE_SIZE])


# ------------------------------------------------------- step 1: centroids --

def num_blocks(seq_len: int, bs: int) -> int:
    return (int(seq_len) + bs - 1) // bs


def build_centroids(keys: np.ndarray, bs: int) -> np.ndarray:
    """Mean-key centroid of every block of `bs` consecutive tokens.

    Block b covers tokens [b*bs, min((b+1)*bs, len)).  The sum runs over the
    block's tokens in token order, in fp64 (one vectorised add per token
    position, across all blocks at once), then divides by the number of
    valid tokens in the block.
    """
    L = keys.shape[0]
    n = num_blocks(L, bs)
    cent = np.zeros((n, HEAD_DIM), dtype=np.float64)
    nfull = L // bs
    if nfull:
        kb = keys[:nfull * bs].reshape(nfull, bs, HEAD_DIM)
        acc = np.zeros((nfull, HEAD_DIM), dtype=np.float64)
        for t in range(bs):
            acc = acc + kb[:, t, :]
        cent[:nfull] = acc / bs
    if n > nfull:                                   # ragged last block
        tail = keys[nfull * bs:]
        acc = np.zeros(HEAD_DIM, dtype=np.float64)
        for t in range(tail.shape[0]):
            acc = acc + tail[t]
        cent[nfull] = acc / tail.shape[0]
    return cent


# ------------------------------------------------------ step 2: INT4 codes --

@dataclass
class QuantizedCentroids:
    codes: np.ndarray      # uint8 [n][128], values 0..15
    scale: np.ndarray      # float32 [128]
    zp: np.ndarray         # int32 [128]


def quantize_centroids(cent: np.ndarray) -> QuantizedCentroids:
    """INT4 asymmetric per-channel quantisation of one head's centroids."""
    n = cent.shape[0]
    codes = np.zeros((n, HEAD_DIM), dtype=np.uint8)
    scale = np.zeros(HEAD_DIM, dtype=np.float32)
    zp = np.zeros(HEAD_DIM, dtype=np.int32)
    if n == 0:
        return QuantizedCentroids(codes, scale, zp)
    mn = np.min(cent, axis=0)
    mx = np.max(cent, axis=0)
    s32 = ((mx - mn) / 15.0).astype(np.float32)
    live = (mx > mn) & (s32 > 0)                  # else: degenerate channel
    s = np.where(live, s32.astype(np.float64), 1.0)
    z = np.clip(np.rint(-mn / s), -2147483648.0, 2147483647.0)
    scale[live] = s32[live]
    zp[live] = z[live].astype(np.int32)
    q = np.clip(np.rint(cent / s[None, :]) + zp.astype(np.float64)[None, :],
                0.0, float(CODE_LEVELS))
    codes[:, live] = q[:, live].astype(np.uint8)
    return QuantizedCentroids(codes, scale, zp)


def append_tail_row(keys: np.ndarray, bs: int, scale: np.ndarray, zp: np.ndarray):
    """Incremental update after appending tokens: the centroid of the block
    that holds the last token, recomputed from that block's keys, and its
    INT4 codes under the per-channel parameters of an earlier build.

    Returns (block index, centroid fp64 [128], codes uint8 [128], number of
    channels whose unclamped code fell outside 0..15, i.e. whose range the
    earlier parameters no longer cover; channels with scale 0 carry no
    information and are not counted).
    """
    L = keys.shape[0]
    b = (L - 1) // bs
    t0 = b * bs
    acc = np.zeros(HEAD_DIM, dtype=np.float64)
    for t in range(t0, L):
        acc = acc + keys[t]
    c = acc / (L - t0)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    z = np.asarray(zp, dtype=np.int64).astype(np.float64)
    live = s > 0
    q = np.where(live, np.rint(c / np.where(live, s, 1.0)) + z, 0.0)
    codes = np.clip(q, 0.0, float(CODE_LEVELS)).astype(np.uint8)
    exceeded = int(np.count_nonzero(live & ((q < 0.0) | (q > CODE_LEVELS))))
    return b, c, codes, exceeded


def dequantize(qc: QuantizedCentroids) -> np.ndarray:
    """(code - zp) * scale, fp64."""
    return (qc.codes.astype(np.float64) - qc.zp.astype(np.float64)[None, :]) \
        * qc.scale.astype(np.float64)[None, :]


def round_bf16(x) -> np.ndarray:
    """fp64 -> nearest bf16 value (ties to even), returned as fp64.

    A bf16 number has 8 significant bits and the exponent range of fp32:
    with x = m * 2**e, 0.5 <= |m| < 1, its spacing near x is 2**(e - 8)
    (2**-133 below the smallest normal 2**-126).  Rounding to a multiple of
    that spacing, ties to even, is exact in fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return np.rint(x / q) * q


def bf16_bits_of(x) -> np.ndarray:
    """Bit patterns (uint16) of values that are exactly bf16."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[n][128] nibbles -> [n][64] bytes; channel 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], HEAD_DIM), dtype=np.uint8)
    out[:, 0::2] = p & 0x0F
    out[:, 1::2] = p >> 4
    return out


# ------------------------------------------------- step 3: block scores --

def group_query(q_heads: np.ndarray, kv_head: int, group: int) -> np.ndarray:
    """Sum of the query vectors of KV head `kv_head`'s GQA group.

    Query head j belongs to KV head j // group (contiguous grouping, GQA).
    """
    qs = q_heads[kv_head * group:(kv_head + 1) * group]
    acc = np.zeros(HEAD_DIM, dtype=np.float64)
    for j in range(qs.shape[0]):
        acc = acc + qs[j]
    return acc


def block_scores(cent_hat: np.ndarray, qbar: np.ndarray) -> np.ndarray:
    """Importance score of every block: qbar . centroid (dot-product
    estimation, Fig. 1)."""
    return cent_hat @ qbar


# -------------------------------------------------- step 4: top-K blocks --

def blocks_per_head(budget_tokens: int, bs: int) -> int:
    """Blocks kept by a head of block size `bs` under a token budget."""
    return max(1, int(budget_tokens) // int(bs))


def select_blocks(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k highest scores, ties to the lower index, ascending."""
    n = scores.shape[0]
    if k >= n:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -scores))   # score desc, then index asc
    return np.sort(order[:k].astype(np.int64))


def selected_tokens(sel: np.ndarray, bs: int, seq_len: int) -> np.ndarray:
    toks = []
    for b in sel:
        t0 = int(b) * bs
        toks.extend(range(t0, min(t0 + bs, int(seq_len))))
    return np.asarray(toks, dtype=np.int64)


# ------------------------------------------- step 5: sparse attention --

def attend(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
           tokens: np.ndarray) -> np.ndarray:
    """Softmax attention of one query over the given token rows (fp64)."""
    if tokens.size == 0:
        return np.zeros(HEAD_DIM, dtype=np.float64)
    k = keys[tokens]
    v = values[tokens]
    z = (k @ q) / math.sqrt(HEAD_DIM)
    z = z - np.max(z)
    p = np.exp(z)
    return (p @ v) / np.sum(p)


# ------------------------------------------------------------ a layer --

@dataclass
class HeadResult:
    seq_len: int
    block_size: int
    centroids: np.ndarray           # fp64 [n][128]
    quant: QuantizedCentroids
    scores: np.ndarray              # fp64 [n]
    k: int                          # blocks kept
    sel: np.ndarray                 # int64, ascending


@dataclass
class LayerResult:
    heads: dict = field(default_factory=dict)    # (s, h) -> HeadResult
    out: np.ndarray = None                       # fp64 [S][Hq][128]


def head_keys_values(layer, s, h):
    L = int(layer.seq_lens[s])
    keys = gather_head_tokens(layer.k_bits, layer.page_table[s], L, h)
    vals = gather_head_tokens(layer.v_bits, layer.page_table[s], L, h)
    return keys, vals


def group_max_scores(cent_hat: np.ndarray, q_heads: np.ndarray, kv_head: int,
                     group: int) -> np.ndarray:
    """Variant aggregation: each block's score is the largest of the group's
    per-head dot products q_j . centroid."""
    qs = q_heads[kv_head * group:(kv_head + 1) * group]
    return np.max(cent_hat @ qs.T, axis=1) if cent_hat.shape[0] else \
        np.zeros(0, dtype=np.float64)


def decode_head(q_heads: np.ndarray, kv_head: int, group: int, chat: np.ndarray,
                keys: np.ndarray, values: np.ndarray, bs: int, seq_len: int,
                budget: int, sel_override=None, aggregate: str = "sum"):
    """Steps 3-5 for one (sequence, KV head) from its (dequantised) centroids.

    aggregate="sum" scores with the group-summed query (the default
    reading); "max" with the largest per-head score (the variant).
    Returns (scores, k, sel, outputs [group][128]).
    """
    if aggregate == "max":
        sc = group_max_scores(chat, q_heads, kv_head, group)
    else:
        qbar = group_query(q_heads, kv_head, group)
        sc = block_scores(chat, qbar)
    k = min(blocks_per_head(budget, bs), chat.shape[0])
    sel = select_blocks(sc, k)
    use = sel if sel_override is None else np.asarray(sel_override, dtype=np.int64)
    toks = selected_tokens(use, bs, seq_len)
    outs = np.zeros((group, HEAD_DIM), dtype=np.float64)
    for i, j in enumerate(range(kv_head * group, (kv_head + 1) * group)):
        outs[i] = attend(q_heads[j], keys, values, toks)
    return sc, k, sel, outs


def run_layer(layer, quantize=True, sel_override=None,
              heads=None, with_attention: bool = True,
              aggregate: str = "sum") -> LayerResult:
    """All five steps for every (sequence, KV head) of a host layer.

    `layer` carries q_bits [S][Hq][128], k_bits / v_bits
    [P][Hkv][16][128] (uint16 bf16 bits), page_table [S][max_pages],
    seq_lens [S], block_size [Hkv] and budget.  `quantize=False` scores the
    fp64 centroids directly (the unquantised variant); `quantize="bf16"`
    scores the centroids rounded to bf16 (the BF16-centroid variant).  `sel_override`
    maps (s, h) -> block list to attend over instead of the oracle's own
    selection.  `heads` restricts the work to some (s, h) pairs.
    """
    S, Hq = layer.q_bits.shape[0], layer.q_bits.shape[1]
    Hkv = len(layer.block_size)
    G = Hq // Hkv
    res = LayerResult(out=np.zeros((S, Hq, HEAD_DIM), dtype=np.float64))
    for s in range(S):
        qf = decode_bf16(layer.q_bits[s])
        for h in range(Hkv):
            if heads is not None and (s, h) not in heads:
                continue
            bs = int(layer.block_size[h])
            L = int(layer.seq_lens[s])
            keys, vals = head_keys_values(layer, s, h)
            cent = build_centroids(keys, bs)
            qc = quantize_centroids(cent)
            if quantize == "bf16":
                chat = round_bf16(cent)
            else:
                chat = dequantize(qc) if quantize else cent
            ov = None if sel_override is None else sel_override[(s, h)]
            sc, k, sel, outs = decode_head(qf, h, G, chat, keys, vals, bs, L,
                                           layer.budget, sel_override=ov,
                                           aggregate=aggregate)
            res.heads[(s, h)] = HeadResult(L, bs, cent, qc, sc, k, sel)
            if with_attention:
                res.out[s, h * G:(h + 1) * G] = outs
    return res
