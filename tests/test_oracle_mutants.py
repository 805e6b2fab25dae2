"""The pins are strong enough: each plausible mistake in the oracle -- a
dropped term, a wrong sign, a wrong index or grouping, a transposed operand,
a rounding or tie-break rule changed -- makes at least one pin of
test_oracle_pins.py fail.

Every mutant below replaces one oracle function, in the oracle module
itself (the other oracle functions call it through the module, as the pins
do), with a version carrying one such mistake; the pins are then run until
one fails.  Nothing here runs on a GPU.
"""

import inspect
import math

import numpy as np
import pytest

import test_oracle_pins as PINS
from oracle import absp_oracle as O

ORIG = {name: getattr(O, name) for name in (
    "decode_bf16", "gather_head_tokens", "build_centroids", "dequantize", "group_query",
    "block_scores", "blocks_per_head", "select_blocks", "selected_tokens", "attend",
    "pack_codes", "round_bf16", "append_tail_row")}


def _pins():
    """(name, callable) of every pin, parametrised ones expanded."""
    out = []
    for name, fn in inspect.getmembers(PINS, inspect.isfunction):
        if not name.startswith("test_") or fn.__module__ != PINS.__name__:
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            out.append((name, fn))
            continue
        argname, values = marks[0].args
        for v in values:
            out.append((f"{name}[{v}]", (lambda f, a, x: lambda: f(**{a: x}))(fn, argname, v)))
    return out


PIN_LIST = _pins()


# ------------------------------------------------------------- mutants --

def _centroid_sum(keys, bs):                       # division by the count dropped
    c = ORIG["build_centroids"](keys, bs)
    L = keys.shape[0]
    cnt = np.array([min(bs, L - b * bs) for b in range(c.shape[0])], dtype=np.float64)
    return c * cnt[:, None]


def _centroid_tail_over_bs(keys, bs):              # ragged tail divided by bs
    c = ORIG["build_centroids"](keys, bs).copy()
    L = keys.shape[0]
    if L % bs:
        c[-1] *= (L % bs) / bs
    return c


def _centroid_shifted(keys, bs):                   # blocks start one token late
    return ORIG["build_centroids"](np.roll(keys, -1, axis=0), bs)


def _quantizer(levels=15.0, zp_sign=-1.0, rnd=np.rint):
    def q(cent):
        n = cent.shape[0]
        codes = np.zeros((n, O.HEAD_DIM), dtype=np.uint8)
        scale = np.zeros(O.HEAD_DIM, dtype=np.float32)
        zp = np.zeros(O.HEAD_DIM, dtype=np.int32)
        if n == 0:
            return O.QuantizedCentroids(codes, scale, zp)
        mn, mx = cent.min(axis=0), cent.max(axis=0)
        s32 = ((mx - mn) / levels).astype(np.float32)
        live = (mx > mn) & (s32 > 0)
        s = np.where(live, s32.astype(np.float64), 1.0)
        z = rnd(zp_sign * mn / s)
        scale[live] = s32[live]
        zp[live] = z[live].astype(np.int32)
        qq = np.clip(rnd(cent / s[None, :]) + zp[None, :], 0, 15)
        codes[:, live] = qq[:, live].astype(np.uint8)
        return O.QuantizedCentroids(codes, scale, zp)
    return q


def _select_ties_high(scores, k):                  # ties to the higher index
    n = scores.shape[0]
    if k >= n:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((-np.arange(n), -scores))
    return np.sort(order[:k].astype(np.int64))


def _select_unsorted(scores, k):                   # list left in score order
    n = scores.shape[0]
    if k >= n:
        return np.arange(n, dtype=np.int64)
    return np.lexsort((np.arange(n), -scores))[:k].astype(np.int64)


def _select_lowest(scores, k):                     # sign of the score flipped
    return ORIG["select_blocks"](-scores, k)


def _attend_unscaled(q, keys, values, tokens):     # 1/sqrt(d) dropped
    return ORIG["attend"](q * math.sqrt(O.HEAD_DIM), keys, values, tokens)


def _attend_keys_as_values(q, keys, values, tokens):   # operands swapped
    return ORIG["attend"](q, keys, keys, tokens)


def _tokens_unclipped(sel, bs, seq_len):           # ragged last block not clipped
    return np.asarray([t for b in sel for t in range(int(b) * bs, int(b) * bs + bs)],
                      dtype=np.int64)


def _gather_no_page_table(pages_bits, row, seq_len, kv_head):   # logical = physical
    t = np.arange(int(seq_len))
    return O.decode_bf16(pages_bits[t // O.PAGE_SIZE, kv_head, t % O.PAGE_SIZE])


def _decode_as_fp16(bits):                          # wrong 16-bit float format
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _pack_swapped(codes):                           # nibble order swapped
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 1::2] | (c[:, 0::2] << 4)).astype(np.uint8)


def _round_bf16_truncate(x):                        # truncation, not nearest
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    b = f.view(np.uint32) & np.uint32(0xFFFF0000)
    return b.view(np.float32).astype(np.float64)


def _append_whole_block(keys, bs, scale, zp):      # tail mean over bs, not valid tokens
    b, c, codes, exc = ORIG["append_tail_row"](keys, bs, scale, zp)
    L = keys.shape[0]
    valid = L - b * bs
    if valid == bs:
        return b, c, codes, exc
    c2 = c * valid / bs
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    live = s > 0
    q = np.where(live, np.rint(c2 / np.where(live, s, 1.0)) + zp, 0.0)
    return b, c2, np.clip(q, 0, 15).astype(np.uint8), exc


MUTANTS = {
    "centroid: sum, not mean": ("build_centroids", _centroid_sum),
    "centroid: ragged tail over bs": ("build_centroids", _centroid_tail_over_bs),
    "centroid: blocks shifted by a token": ("build_centroids", _centroid_shifted),
    "quantise: 16 steps, not 15": ("quantize_centroids", _quantizer(levels=16.0)),
    "quantise: zero point sign": ("quantize_centroids", _quantizer(zp_sign=1.0)),
    "quantise: ties away from zero": ("quantize_centroids",
                                      _quantizer(rnd=lambda x: np.floor(x + 0.5))),
    "dequantise: zero point dropped": ("dequantize",
                                       lambda qc: qc.codes.astype(np.float64) *
                                       qc.scale.astype(np.float64)[None, :]),
    "score: first query head only": ("group_query", lambda q, h, g: q[h * g].copy()),
    "score: interleaved GQA grouping": ("group_query",
                                        lambda q, h, g: q[h::q.shape[0] // g].sum(axis=0)),
    "score: half of the channels": ("block_scores",
                                    lambda chat, qbar: chat[:, :64] @ qbar[:64]),
    "top-K: ties to the higher index": ("select_blocks", _select_ties_high),
    "top-K: not ascending": ("select_blocks", _select_unsorted),
    "top-K: lowest scores": ("select_blocks", _select_lowest),
    "top-K: budget in pages, not blocks": ("blocks_per_head",
                                           lambda b, bs: max(1, int(b) // 16)),
    "top-K: one block too many": ("blocks_per_head", lambda b, bs: max(1, int(b) // int(bs)) + 1),
    "tokens: ragged block not clipped": ("selected_tokens", _tokens_unclipped),
    "attention: 1/sqrt(d) dropped": ("attend", _attend_unscaled),
    "attention: keys as values": ("attend", _attend_keys_as_values),
    "gather: page table ignored": ("gather_head_tokens", _gather_no_page_table),
    "input: bf16 read as fp16": ("decode_bf16", _decode_as_fp16),
    "codes: nibble order swapped": ("pack_codes", _pack_swapped),
    "bf16 centroids: truncation": ("round_bf16", _round_bf16_truncate),
    "append: tail mean over bs": ("append_tail_row", _append_whole_block),
}


def test_every_pin_passes_unmutated():
    for name, fn in PIN_LIST:
        fn()


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for name, pin in PIN_LIST:
        try:
            pin()
        except Exception as e:   # an assertion, or the mutant breaking a pin outright
            caught.append((name, type(e).__name__))
            break
    assert caught, f"no pin fails for the mutant '{mutant}'"
