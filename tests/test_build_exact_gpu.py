"""The centroid build's exact fast path against the token-order fp64
definition, bit for bit.

The build kernels sum a page's 16 keys per channel in fp32, rounded down
and rounded up, and keep the sum when the two agree (both are then exact);
a block whose keys span more than 39 binades, or hold a zero, subnormal,
infinite or NaN key, is summed again in token order.  The key mixes below
are chosen so that every branch runs: plain normal keys (fast path),
keys scaled by 2^k for k in [-12, 12] (fp32 page sums inexact, block
within the span), k in [-60, 60] (block outside the span), exact zeros of
both signs, subnormal keys, pairs that cancel exactly (zero sums, whose
sign must be +0), and keys near the top of the bf16 range (fp32 page sums
that overflow).  The fp64 centroids the build leaves in its workspace are
compared with the oracle's token-order sums, and the one-call build with
the two calls, for INT4 codes and bf16 rows."""

import numpy as np
import pytest
import torch

from block_sparse_attention_kv_b200 import synth
from oracle import absp_oracle as O

pytestmark = pytest.mark.gpu

KINDS = ["plain", "spread12", "spread60", "zeros", "subnormal", "cancel", "huge"]
WORKLOAD = synth.custom("exact_sums", 3, 6, 3, [2085, 1000, 80], [16, 32, 64], 256, seed=77)


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, pipeline
    return abi, pipeline


def _keys(kind: str, shape, rng) -> np.ndarray:
    x = rng.standard_normal(shape).astype(np.float32)
    if kind == "spread12":
        x *= np.exp2(rng.integers(-12, 13, shape)).astype(np.float32)
    elif kind == "spread60":
        x *= np.exp2(rng.integers(-60, 61, shape)).astype(np.float32)
    elif kind == "zeros":
        m = rng.random(shape) < 0.03
        x[m] = 0.0
        x[m & (rng.random(shape) < 0.5)] = -0.0
    elif kind == "subnormal":
        m = rng.random(shape) < 0.05
        x[m] *= np.float32(2.0 ** -130)
    elif kind == "cancel":
        x[1::2] = -x[0::2]
    elif kind == "huge":
        x *= np.float32(2.0 ** 125)
    return x


def _layer(kind: str):
    """The workload's layer with its valid key rows replaced by `kind` keys
    (rows past each sequence's length keep their NaN fill)."""
    d = synth.make_layer(WORKLOAD, 0, "cuda")
    rng = np.random.default_rng(1000 + KINDS.index(kind))
    Hkv, D, P = d.num_kv_heads, 128, synth.PAGE_SIZE
    for s in range(d.num_seqs):
        L = int(d.seq_lens[s])
        npg = (L + P - 1) // P
        if npg == 0:
            continue
        kk = _keys(kind, (npg * P, Hkv, D), rng)
        kk[L:] = np.nan
        kb = torch.from_numpy(kk).to("cuda").to(torch.bfloat16)
        ids = d.page_table[s, :npg].long()
        d.k_pages[ids] = kb.view(npg, P, Hkv, D).permute(0, 2, 1, 3)
    return d


def _ws_centroids(abi, dl) -> torch.Tensor:
    d = dl.data
    off = 256 + d.num_seqs * d.num_kv_heads * 128 * 2 * 8
    return dl.build_ws[off:].view(torch.float64).view(-1, 128)


@pytest.mark.parametrize("kind", KINDS)
def test_fp64_centroids_are_the_token_order_sums(lib, kind):
    abi, pipeline = lib
    d = _layer(kind)
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids(keep_ws=True)
    torch.cuda.synchronize()
    gpu = _ws_centroids(abi, dl).cpu().numpy().view(np.uint64)
    host = synth.host_layer(d)
    checked = 0
    for s in range(d.num_seqs):
        L = int(host.seq_lens[s])
        for h in range(d.num_kv_heads):
            bs = int(d.block_size[h])
            keys = O.gather_head_tokens(host.k_bits, host.page_table[s], L, h)
            want = O.build_centroids(keys, bs).view(np.uint64)
            r0 = abi.absp_centroid_row_offset(dl.kv, s, h)
            got = gpu[r0:r0 + want.shape[0]]
            bad = np.argwhere(got != want)
            assert bad.size == 0, (kind, s, h, bad[:4].tolist())
            checked += want.size
    assert checked > 0


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("fmt", [0, 1], ids=["int4", "bf16"])
def test_one_call_build_equals_two_calls(lib, kind, fmt):
    abi, pipeline = lib
    d = _layer(kind)
    a = pipeline.DeviceLayer(d, fmt=fmt)
    b = pipeline.DeviceLayer(d, fmt=fmt)
    a.build_centroids()
    b.cent.codes.fill_(0xAB)
    b.build_centroids(fused=True)
    torch.cuda.synchronize()
    for s in range(d.num_seqs):
        L = int(d.seq_lens[s])
        for h in range(d.num_kv_heads):
            n = (L + int(d.block_size[h]) - 1) // int(d.block_size[h])
            assert torch.equal(a.codes_of(s, h, n), b.codes_of(s, h, n)), (kind, s, h)
    if fmt == 0:
        assert torch.equal(a.cent.scale.view(torch.int32), b.cent.scale.view(torch.int32))
        assert torch.equal(a.cent.zp, b.cent.zp)
