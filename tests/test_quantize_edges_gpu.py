"""The quantise step on centroids placed at its rounding edges, against the
oracle, bit for bit.

The kernel codes a centroid as rint(c * (1/scale)) when that product is
below 2^20 and at least 2^-28 from every half-integer, and as the exact
rint(c / scale) otherwise.  Here the fp64 centroids are written straight
into the build workspace (its layout is part of the header: error word,
order-mapped min / max keys, then the rows) and absp_quantize_centroids
codes them; the values sit on half-integers of c / scale, a few ulps to
either side of them, 2^-29 .. 2^-27 away (both sides of the 2^-28 margin),
and at quotients around 2^20 and far beyond, so that both paths and ties
(round half to even) are taken."""

import numpy as np
import pytest
import torch

from block_sparse_attention_kv_b200 import synth
from oracle import absp_oracle as O

pytestmark = pytest.mark.gpu

WORKLOAD = synth.custom("quant_edges", 2, 4, 2, [4096, 1500], [16, 32], 256, seed=91)


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, pipeline
    return abi, pipeline


def _ord_key(x: np.ndarray) -> np.ndarray:
    """Order-mapped fp64 key (min over keys = min over values)."""
    u = x.astype(np.float64).view(np.uint64)
    neg = (u >> np.uint64(63)) != 0
    return np.where(neg, ~u, u | np.uint64(1 << 63))


def _edge_rows(n: int, rng) -> np.ndarray:
    """n rows x 128 channels; each channel has its own range and scale, the
    rows placed at and around the rounding edges of c / scale."""
    rows = np.empty((n, 128), dtype=np.float64)
    for ch in range(128):
        kind = ch % 4
        if kind == 3:
            # quotients near and far beyond 2^20: the minimum far from 0
            lo = float(rng.choice([2.0 ** 16, 2.0 ** 21, 2.0 ** 40])) * rng.uniform(1, 2)
        else:
            lo = rng.uniform(-3, 3)
        span = float(rng.choice([1e-3, 0.7, 15.0, 1e3]))
        hi = lo + span
        # the scale exactly as the method forms it from this min and max
        s = float(np.float32((hi - lo) / 15.0))
        col = []
        for i in range(n):
            k = int(rng.integers(0, 16)) + np.floor(lo / s)
            half = (k + 0.5) * s
            off = [0.0, np.spacing(half), -np.spacing(half), 2 * np.spacing(half),
                   s * 2.0 ** -29, -s * 2.0 ** -29, s * 2.0 ** -27, -s * 2.0 ** -27,
                   s * rng.uniform(-0.5, 0.5)][i % 9]
            col.append(half + off)
        col = np.clip(np.asarray(col), lo, hi)
        # pin the channel's min and max (the scale above is theirs)
        col[0] = lo
        if n > 1:
            col[1] = hi
        rows[:, ch] = col
    return rows


def test_codes_at_the_rounding_edges_match_the_oracle(lib):
    abi, pipeline = lib
    d = synth.make_layer(WORKLOAD, 0, "cuda")
    dl = pipeline.DeviceLayer(d)
    ws = abi.alloc_workspace(abi.absp_build_workspace_size(dl.kv), "cuda")
    S, Hkv = d.num_seqs, d.num_kv_heads
    pairs = S * Hkv
    rng = np.random.default_rng(5)
    mins = np.zeros((pairs, 128), dtype=np.uint64)
    maxs = np.zeros((pairs, 128), dtype=np.uint64)
    rows_all = {}
    cent_off = 256 + pairs * 128 * 2 * 8
    cent = ws[cent_off:].view(torch.float64).view(-1, 128)
    for s in range(S):
        L = int(d.seq_lens[s])
        for h in range(Hkv):
            bs = int(d.block_size[h])
            n = (L + bs - 1) // bs
            r = _edge_rows(n, rng)
            rows_all[(s, h)] = r
            r0 = abi.absp_centroid_row_offset(dl.kv, s, h)
            cent[r0:r0 + n] = torch.from_numpy(r).to("cuda")
            mins[s * Hkv + h] = _ord_key(r.min(axis=0))
            maxs[s * Hkv + h] = _ord_key(-r.max(axis=0))
    keys = np.concatenate([mins.ravel(), maxs.ravel()]).view(np.int64)
    ws[256:cent_off].view(torch.int64).copy_(torch.from_numpy(keys).to("cuda"))
    abi.absp_quantize_centroids(dl.kv, ws, dl.cent, None)
    st, detail = abi.absp_check_device_error(ws, None)
    assert st == abi.ABSP_OK, (st, detail)
    checked = 0
    for (s, h), r in rows_all.items():
        want = O.quantize_centroids(r)
        n = r.shape[0]
        got = O.unpack_codes(dl.codes_of(s, h, n).cpu().numpy())
        scale, zp = dl.params_of(s, h)
        assert np.array_equal(scale.cpu().numpy().view(np.uint32), want.scale.view(np.uint32)), (s, h)
        assert np.array_equal(zp.cpu().numpy(), want.zp), (s, h)
        bad = np.argwhere(got != want.codes)
        assert bad.size == 0, (s, h, bad[:4].tolist(), r[tuple(bad[0])] if bad.size else None)
        checked += n * 128
    assert checked > 0
