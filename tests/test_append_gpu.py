"""GPU parity of the incremental centroid update (absp_append_centroids).

The store is built at a shorter length, then the sequence grows one token at
a time (the pages already hold the tokens; raising seq_lens appends them).
After every append the tail row and the count of channels out of the
earlier range must equal the oracle's, and every other row must stay as
built.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_kv_b200 import synth
from oracle import absp_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, pipeline
    return abi, pipeline


def _tail_want(hl, s, h, L, scale, zp, fmt):
    keys = O.gather_head_tokens(hl.k_bits, hl.page_table[s], L, h)
    if fmt == 1:                       # BF16 rows: no per-channel parameters
        scale, zp = np.ones(128, np.float32), np.zeros(128, np.int32)
    b, c, codes, exc = O.append_tail_row(keys, int(hl.block_size[h]), scale, zp)
    if fmt == 1:
        return b, O.bf16_bits_of(O.round_bf16(c)).view(np.uint8), 0
    return b, O.pack_codes(codes[None, :])[0], exc


@pytest.mark.parametrize("fmt", [0, 1])
def test_append_tokens_one_by_one(lib, fmt):
    abi, pipeline = lib
    full = [700, 1500]
    w = synth.custom("append", 2, 8, 2, full, [16, 64], 256, seed=70)
    d = synth.make_layer(w, 0, "cuda")
    hl = synth.host_layer(d)
    start = [f - 40 for f in full]
    d.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    dl = pipeline.DeviceLayer(d, fmt=fmt)
    dl.build_centroids()
    torch.cuda.synchronize()
    base = dl.cent.codes.clone()
    params = {(s, h): tuple(t.cpu().numpy() for t in dl.params_of(s, h))
              for s in range(2) for h in range(2)}
    exceeded = torch.full((2, 2), -1, dtype=torch.int32, device="cuda")
    touched = set()
    rb = 256 if fmt == 1 else 64
    for step in range(1, 41):
        lens = [x + step for x in start]
        d.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
        abi.absp_append_centroids(dl.kv, dl.cent, exceeded, dl.ws)
        dl.check()
        exc = exceeded.cpu().numpy()
        for s in range(2):
            for h in range(2):
                scale, zp = params[(s, h)]
                b, want, wexc = _tail_want(hl, s, h, lens[s], scale, zp, fmt)
                row = dl.codes_of(s, h, b + 1)[b].cpu().numpy()
                assert np.array_equal(row, want), (step, s, h, b)
                assert exc[s, h] == wexc, (step, s, h)
                touched.add(abi.absp_centroid_row_offset(dl.kv, s, h) + b)
    # every row not appended to is unchanged
    now = dl.cent.codes.view(-1, rb).cpu()
    was = base.view(-1, rb).cpu()
    keep = torch.ones(now.shape[0], dtype=torch.bool)
    keep[list(touched)] = False
    assert torch.equal(now[keep], was[keep])


def test_append_flags_channels_beyond_the_range(lib):
    abi, pipeline = lib
    w = synth.custom("append_big", 1, 4, 1, [300], [32], 128, seed=71, planted_blocks=0)
    d = synth.make_layer(w, 0, "cuda")
    d.seq_lens.fill_(299)
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    # token 299 gets a huge value in channels 0..9: its block's mean leaves
    # the range of the earlier build there
    pg = int(d.page_table[0, 299 // 16])
    d.k_pages[pg, 0, 299 % 16, :10] = 500.0
    d.seq_lens.fill_(300)
    hl = synth.host_layer(d)
    exceeded = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    abi.absp_append_centroids(dl.kv, dl.cent, exceeded, dl.ws)
    dl.check()
    scale, zp = (t.cpu().numpy() for t in dl.params_of(0, 0))
    b, want, wexc = _tail_want(hl, 0, 0, 300, scale, zp, 0)
    # the 10 forced channels at least (others may leave the range too when
    # this short tail block was a channel's extreme)
    assert wexc >= 10
    assert int(exceeded.item()) == wexc
    assert np.array_equal(dl.codes_of(0, 0, b + 1)[b].cpu().numpy(), want)
