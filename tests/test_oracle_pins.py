"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks one step against a closed form, a hand-worked example, an
exact-rational or brute-force computation, a library routine the step
reduces to in a special case, or an invariant of the method (AB-Sparse,
arXiv 2605.12110: Fig. 1 pipeline, Fig. 8 INT4 asymmetric per-channel
centroids, Fig. 9 equal token budget across block sizes).
"""

import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import absp_oracle as O
from block_sparse_attention_kv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------ bf16 input --

def test_decode_bf16_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3FC0, 0x4049, 0x0001, 0x8000, 0x7F80,
                     0x0080], dtype=np.uint16)
    want = [1.0, -2.0, 1.5, 3.140625, 2.0 ** -133, -0.0, math.inf, 2.0 ** -126]
    got = O.decode_bf16(bits)
    for g, w in zip(got, want):
        assert g == w
    assert math.copysign(1.0, got[5]) == -1.0


def test_gather_follows_page_table():
    # 3 physical pages, 2 heads; logical page i of the sequence is physical
    # page perm[i]; every slot holds a distinct small integer id.
    P, H = 3, 2
    perm = np.array([2, 0, 1], dtype=np.int32)
    vals = np.zeros((P, H, 16, 128), dtype=np.float32)
    for p in range(P):
        for h in range(H):
            for t in range(16):
                vals[p, h, t, :] = p * 100 + h * 40 + t    # exact in bf16? <=255 ok
    vals = np.minimum(vals, 255)
    bits = _bf16_bits(vals)
    L = 40
    got = O.gather_head_tokens(bits, perm, L, 1)
    for t in range(L):
        want = min(perm[t // 16] * 100 + 40 + t % 16, 255)
        assert np.all(got[t] == want)


# -------------------------------------------------------- step 1: centroid --

def test_centroid_block_size_one_is_identity():
    rng = np.random.default_rng(0)
    keys = O.decode_bf16(_bf16_bits(rng.standard_normal((37, 128))))
    assert np.array_equal(O.build_centroids(keys, 1), keys)


def test_centroid_constant_block_and_ragged_tail():
    keys = np.zeros((5, 128))
    for t in range(5):
        keys[t] = t                   # block 0 = tokens 0..3, block 1 = token 4
    c = O.build_centroids(keys, 4)
    assert c.shape == (2, 128)
    assert np.all(c[0] == 1.5) and np.all(c[1] == 4.0)
    const = np.full((64, 128), -2.25)
    assert np.all(O.build_centroids(const, 32) == -2.25)


@pytest.mark.parametrize("bs", [16, 32, 64])
def test_centroid_equals_exact_rational_mean(bs):
    # bf16 inputs with a +6 outlier channel; the fp64 token-order sum is
    # exact, so the centroid must be the correctly rounded rational mean.
    rng = np.random.default_rng(bs)
    L = 3 * bs + 5
    x = rng.standard_normal((L, 128))
    x[:, 7] += 6.0
    keys = O.decode_bf16(_bf16_bits(x))
    c = O.build_centroids(keys, bs)
    for b in range(c.shape[0]):
        t0, t1 = b * bs, min((b + 1) * bs, L)
        for d in (0, 7, 64, 127):
            exact = sum((Fraction(float(keys[t, d])) for t in range(t0, t1)),
                        Fraction(0)) / (t1 - t0)
            assert c[b, d] == float(exact)


# ------------------------------------------------------- step 2: INT4 codes --

def _one_channel(vals):
    cent = np.zeros((len(vals), 128))
    cent[:, 0] = vals
    return O.quantize_centroids(cent)


def test_quantize_hand_examples():
    # range 15 -> scale exactly 1: 2.5 and 3.5 test round-half-to-even.
    q = _one_channel([0.0, 2.5, 3.5, 15.0])
    assert q.scale[0] == np.float32(1.0) and q.zp[0] == 0
    assert list(q.codes[:, 0]) == [0, 2, 4, 15]
    # negative minimum -> zero point 3
    q = _one_channel([-3.0, 0.0, 12.0])
    assert q.scale[0] == 1.0 and q.zp[0] == 3
    assert list(q.codes[:, 0]) == [0, 3, 15]
    # an outlier channel that excludes 0: scale = fp32(0.1), zp = -55
    q = _one_channel([5.5, 6.25, 7.0])
    assert q.scale[0] == np.float32(0.1)
    assert q.zp[0] == -55
    assert list(q.codes[:, 0]) == [0, 7, 15]
    # the other 127 channels are constant zero: degenerate
    assert np.all(q.scale[1:] == 0) and np.all(q.zp[1:] == 0)
    assert np.all(q.codes[:, 1:] == 0)


def test_quantize_degenerate_single_block():
    q = O.quantize_centroids(np.full((1, 128), 3.0))
    assert np.all(q.scale == 0) and np.all(q.zp == 0) and np.all(q.codes == 0)


def test_dequantize_error_bound_and_endpoints():
    rng = np.random.default_rng(5)
    cent = rng.standard_normal((700, 128)) * 0.25
    cent[:, :4] += 6.0                               # outlier channels
    cent[:, 50] *= 1e-3                              # narrow channel
    q = O.quantize_centroids(cent)
    deq = O.dequantize(q)
    s = q.scale.astype(np.float64)
    assert np.all(s > 0)
    err = np.abs(deq - cent)
    assert np.all(err <= s[None, :] * (0.5 + 1e-6))
    # the minimum of each channel maps to code 0, the maximum to 15
    assert np.all(q.codes[np.argmin(cent, axis=0), np.arange(128)] == 0)
    assert np.all(q.codes[np.argmax(cent, axis=0), np.arange(128)] >= 14)
    assert np.mean(q.codes.max(axis=0) == 15) > 0.99
    assert q.codes.max() <= 15


def test_code_is_nearest_level_brute_force():
    # with a power-of-two scale every step is exact, so code must be the
    # index of the nearest representable level (ties to the even integer).
    rng = np.random.default_rng(9)
    vals = np.round(rng.uniform(-4, 11, size=50) * 4) / 4
    vals[0], vals[1] = -4.0, 11.0                    # range 15 -> scale 1
    q = _one_channel(vals)
    assert q.scale[0] == 1.0
    for i, v in enumerate(vals):
        best = min(range(16), key=lambda c: (abs((c - q.zp[0]) - v),
                                             (c - q.zp[0]) % 2))
        assert q.codes[i, 0] == best


def test_append_tail_row_equals_rebuild_row_within_range():
    # appending tokens and re-quantising the tail block with the old
    # parameters gives the full rebuild's row whenever the new centroid stays
    # inside the old per-channel range
    rng = np.random.default_rng(12)
    keys = O.decode_bf16(_bf16_bits(rng.standard_normal((200, 128))))
    bs = 16
    old = O.quantize_centroids(O.build_centroids(keys[:180], bs))
    b, c, codes, exc = O.append_tail_row(keys[:181], bs, old.scale, old.zp)
    assert b == 11                                   # token 180 is in block 11
    full = O.build_centroids(keys[:181], bs)
    assert np.array_equal(c, full[11])
    cd = old.codes.astype(np.float64)
    s = old.scale.astype(np.float64)
    want = np.clip(np.rint(full[11] / s) + old.zp, 0, 15)
    assert np.array_equal(codes, want.astype(np.uint8))
    # a single-token block closes the previous one: block 12 holds token 192
    b2, c2, _, _ = O.append_tail_row(keys[:193], bs, old.scale, old.zp)
    assert b2 == 12 and np.array_equal(c2, keys[192])
    assert exc >= 0


def test_append_tail_row_flags_out_of_range_channels():
    keys = np.zeros((17, 128))
    keys[:16, 0] = np.linspace(-1.0, 1.0, 16)        # block 0
    keys[:16, 1] = 0.5
    scale = np.full(128, np.float32(0.1))
    zp = np.full(128, 5, dtype=np.int32)
    keys[16, 0] = 100.0                              # far above code 15
    keys[16, 1] = -0.2                               # code 3: inside
    b, c, codes, exc = O.append_tail_row(keys, 16, scale, zp)
    assert b == 1 and codes[0] == 15 and codes[1] == 3 and exc == 1
    scale[0] = 0.0                                   # degenerate channel: not counted
    assert O.append_tail_row(keys, 16, scale, zp)[3] == 0


def test_pack_nibble_order_round_trip():
    codes = np.arange(128, dtype=np.uint8).reshape(1, 128) % 16
    p = O.pack_codes(codes)
    assert p.shape == (1, 64)
    assert p[0, 0] == 0x10 and p[0, 1] == 0x32 and p[0, 7] == 0xFE
    assert np.array_equal(O.unpack_codes(p), codes)


def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0]])
    x32 = x.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x32.astype(np.float64)), want)


def test_round_bf16_has_no_double_rounding():
    # halfway between 1 and 1+2^-7 plus a tail that fp32 cannot hold: the
    # correct result rounds up; rounding through fp32 first would tie to 1.0
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert O.round_bf16(x) == 1.0 + 2.0 ** -7
    assert O.round_bf16(1.0 + 2.0 ** -8) == 1.0            # exact tie -> even
    assert O.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.round_bf16(2.0 ** -133 * 0.75) == 2.0 ** -133  # subnormal spacing
    assert O.bf16_bits_of(np.array([1.0, -2.0]))[1] == 0xC000


# ------------------------------------------------------- step 3: scores --

def test_group_query_and_score_equal_sum_of_per_head_dots():
    # bs = 1 without quantisation: a block is one token, and the score of the
    # GQA group sum equals the sum over the group's heads of q_j . k_t.
    rng = np.random.default_rng(3)
    G, Hkv = 4, 3
    q = rng.standard_normal((G * Hkv, 128))
    keys = rng.standard_normal((20, 128))
    for h in range(Hkv):
        sc = O.block_scores(O.build_centroids(keys, 1), O.group_query(q, h, G))
        want = [sum(float(np.dot(q[j], keys[t])) for j in range(h * G, h * G + G))
                for t in range(20)]
        np.testing.assert_allclose(sc, want, rtol=1e-12, atol=1e-12)


def test_group_max_is_max_of_per_head_dots_and_sum_bound():
    rng = np.random.default_rng(14)
    G, Hkv = 4, 2
    q = rng.standard_normal((G * Hkv, 128))
    c = rng.standard_normal((25, 128))
    for h in range(Hkv):
        got = O.group_max_scores(c, q, h, G)
        for b in range(25):
            dots = [float(np.dot(q[j], c[b])) for j in range(h * G, h * G + G)]
            assert got[b] == pytest.approx(max(dots), rel=1e-12, abs=1e-12)
        # the summed-query score never exceeds G times the max
        assert np.all(O.block_scores(c, O.group_query(q, h, G)) <= G * got + 1e-9)
    # with a group of one the two aggregations coincide
    np.testing.assert_allclose(O.group_max_scores(c, q, 3, 1),
                               O.block_scores(c, O.group_query(q, 3, 1)), rtol=1e-12)


def test_score_is_linear_in_query():
    rng = np.random.default_rng(4)
    c = rng.standard_normal((30, 128))
    qb = rng.standard_normal(128)
    assert np.array_equal(O.block_scores(c, 2.0 * qb), 2.0 * O.block_scores(c, qb))


def test_planted_blocks_are_selected_on_tiny_workload():
    # The planted spans (keys + 2 qbar/|qbar|) must rank at the top: a wrong
    # sign, transposed operand or wrong group would lose them.
    w = synth.WORKLOADS["tiny_8k"]
    d = synth.make_layer(w, 0, "cpu")
    hl = synth.host_layer(d)
    res = O.run_layer(hl, with_attention=False)
    for (s, h), hr in res.heads.items():
        bs = hr.block_size
        planted = set()
        for st in d.plan.planted[s][h]:
            planted.update(range(int(st) // bs, (int(st) + 64) // bs))
        assert planted <= set(hr.sel.tolist()), (s, h)


# ------------------------------------------------------- step 4: top-K --

def test_topk_matches_brute_force_subsets():
    rng = np.random.default_rng(11)
    for trial in range(60):
        n = int(rng.integers(1, 11))
        k = int(rng.integers(1, 5))
        sc = rng.integers(-3, 4, size=n).astype(np.float64)   # many ties
        got = O.select_blocks(sc, min(k, n))
        best = None
        for sub in itertools.combinations(range(n), min(k, n)):
            key = (-sum(sc[list(sub)]), sub)                # max sum, then lexicographic
            if best is None or key < best:
                best = key
        assert tuple(got.tolist()) == best[1]


def test_fig9_equal_token_budget_golden():
    rows = [list(map(int, ln.split())) for ln in
            open(os.path.join(GOLDEN, "fig9_equal_budget.txt"))
            if ln.strip() and not ln.startswith("#")]
    for page, budget, bs, kept, pages in rows:
        assert O.blocks_per_head(budget, bs) == kept
        assert kept * bs // page == pages


# ------------------------------------------------------- step 5: attention --

def _sdpa(q, k, v, mask=None):
    # library routine: PyTorch scaled-dot-product attention in fp64 (CPU)
    qt = torch.as_tensor(q)[None, None, None, :]
    kt = torch.as_tensor(k)[None, None]
    vt = torch.as_tensor(v)[None, None]
    m = None if mask is None else torch.as_tensor(mask)[None, None, None, :]
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=m)[0, 0, 0].numpy()


def _small_layer(lens, bs, budget, G=2, seed=0):
    w = synth.custom("pin", len(lens), G * len(bs), len(bs), lens, bs, budget,
                     seed, planted_blocks=2, spare_pages=3)
    return synth.make_layer(w, 0, "cpu")


def test_full_budget_reproduces_dense_attention():
    d = _small_layer([200, 77], [16, 32], budget=4096)
    hl = synth.host_layer(d)
    res = O.run_layer(hl)
    G = 2
    for s in range(2):
        qf = O.decode_bf16(hl.q_bits[s])
        for h in range(2):
            keys, vals = O.head_keys_values(hl, s, h)
            assert len(res.heads[(s, h)].sel) == O.num_blocks(hl.seq_lens[s],
                                                              hl.block_size[h])
            for j in range(h * G, h * G + G):
                np.testing.assert_allclose(res.out[s, j], _sdpa(qf[j], keys, vals),
                                           rtol=1e-10, atol=1e-12)


def test_block_size_one_unquantised_is_exact_token_topk():
    # With one-token blocks and no quantisation, the method is exact
    # top-B-token attention by the group-summed query (brute force).
    rng = np.random.default_rng(21)
    L, B, G = 300, 40, 3
    keys = O.decode_bf16(_bf16_bits(rng.standard_normal((L, 128))))
    vals = O.decode_bf16(_bf16_bits(rng.standard_normal((L, 128))))
    q = O.decode_bf16(_bf16_bits(rng.standard_normal((G, 128))))
    cent = O.build_centroids(keys, 1)
    qbar = O.group_query(q, 0, G)
    sel = O.select_blocks(O.block_scores(cent, qbar), O.blocks_per_head(B, 1))
    toks = O.selected_tokens(sel, 1, L)
    dots = np.array([sum(float(np.dot(q[j], keys[t])) for j in range(G))
                     for t in range(L)])
    top = sorted(range(L), key=lambda t: (-dots[t], t))[:B]
    assert sorted(top) == toks.tolist()
    mask = np.full(L, -np.inf)
    mask[top] = 0.0
    for j in range(G):
        np.testing.assert_allclose(O.attend(q[j], keys, vals, toks),
                                   _sdpa(q[j], keys, vals, mask),
                                   rtol=1e-10, atol=1e-12)


def test_attention_shift_invariance_and_masking():
    d = _small_layer([150], [32], budget=64, seed=3)
    hl = synth.host_layer(d)
    # pages hold NaN past the sequence end: outputs must stay finite
    res = O.run_layer(hl)
    assert np.all(np.isfinite(res.out))
    keys, vals = O.head_keys_values(hl, 0, 0)
    toks = O.selected_tokens(res.heads[(0, 0)].sel, 32, 150)
    assert toks.max() < 150
    q = O.decode_bf16(hl.q_bits[0, 0])
    shift = np.linspace(-1, 1, 128)
    np.testing.assert_allclose(O.attend(q, keys, vals + shift, toks),
                               O.attend(q, keys, vals, toks) + shift,
                               rtol=1e-12, atol=1e-12)


def test_selected_tokens_clip_ragged_last_block():
    t = O.selected_tokens(np.array([0, 4]), 32, 140)
    assert t.tolist() == list(range(32)) + list(range(128, 140))
