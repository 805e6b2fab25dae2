"""Steps 1-2 in one call (absp_build_quantize_centroids) against the two
separate calls, bit for bit, and against the oracle on the full
Llama-shaped layer; heads up to 8192 rows (one 128K sequence at block
size 16).  The BF16 store takes one launch that writes the rows directly."""

import numpy as np
import pytest
import torch

from block_sparse_attention_kv_b200 import synth
from oracle import absp_oracle as O
from oracle import parity as PR

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, pipeline
    return abi, pipeline


CASES = [
    synth.WORKLOADS["tiny_8k"],
    synth.custom("fused_ragged", 5, 12, 3, [4097, 1, 0, 1000, 17], [16, 32, 64], 256, seed=41),
    synth.custom("fused_uniform64", 2, 8, 2, [32768, 5000], [64, 64], 1024, seed=42),
    synth.WORKLOADS["llama31_8b_32k"],
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
@pytest.mark.parametrize("fmt", [0, 1], ids=["int4", "bf16"])
def test_fused_equals_two_calls(lib, w, fmt):
    abi, pipeline = lib
    d = synth.make_layer(w, 0, "cuda")
    a = pipeline.DeviceLayer(d, fmt=fmt)
    b = pipeline.DeviceLayer(d, fmt=fmt)
    a.build_centroids()
    b.cent.codes.fill_(0xAB)                 # stale contents must be overwritten
    if fmt == 0:
        b.cent.scale.fill_(-1.0)
        b.cent.zp.fill_(-7)
    b.build_centroids(fused=True)
    torch.cuda.synchronize()
    for s in range(d.num_seqs):
        L = int(d.seq_lens[s])
        for h in range(d.num_kv_heads):
            n = (L + int(d.block_size[h]) - 1) // int(d.block_size[h])
            assert torch.equal(a.codes_of(s, h, n), b.codes_of(s, h, n)), (s, h)
    if fmt == 0:
        assert torch.equal(a.cent.scale.view(torch.int32), b.cent.scale.view(torch.int32))
        assert torch.equal(a.cent.zp, b.cent.zp)


def test_fused_on_heads_of_8192_rows(lib):
    abi, pipeline = lib
    # one 128K sequence with block size 16: 8192 rows in one head
    w = synth.custom("fused_fallback", 1, 8, 2, [131072], [16, 64], 2048, seed=43)
    d = synth.make_layer(w, 0, "cuda")
    a = pipeline.DeviceLayer(d)
    b = pipeline.DeviceLayer(d)
    a.build_centroids()
    b.build_centroids(fused=True)
    torch.cuda.synchronize()
    assert torch.equal(a.cent.codes, b.cent.codes)
    assert torch.equal(a.cent.scale.view(torch.int32), b.cent.scale.view(torch.int32))
    assert torch.equal(a.cent.zp, b.cent.zp)


def test_fused_matches_the_oracle_on_the_llama_layer(lib):
    abi, pipeline = lib
    d = synth.make_layer(synth.WORKLOADS["llama31_8b_32k"], 1, "cuda")
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids(fused=True)
    torch.cuda.synchronize()
    res = O.run_layer(synth.host_layer(d), with_attention=False)
    rep = PR.Report()
    for h in range(d.num_kv_heads):
        hr = res.heads[(0, h)]
        n = hr.centroids.shape[0]
        scale, zp = dl.params_of(0, h)
        PR.compare_codes(rep, hr, dl.codes_of(0, h, n).cpu().numpy(), scale.cpu().numpy(),
                         zp.cpu().numpy())
        rep.heads += 1
    assert rep.code_mismatch == 0 and rep.param_mismatch == 0, rep.notes[:5]


def test_one_call_codes_on_exact_half_steps(lib):
    """Steps 1-2 on exact ties of c / scale, built from the keys: every
    block holds one key value per channel, placed at j / 2 steps of a
    per-channel step e (min at j = 0, max at j = 30, so scale = e and
    c / scale = offset + j / 2), so odd j give exact half-integers (about
    half of the 40,960 codes), which round half to even.  The one call
    must equal the two calls and the oracle bit for bit."""
    abi, pipeline = lib
    w = synth.custom("half_steps", 1, 8, 2, [4096], [16, 64], 1024, seed=44)
    d = synth.make_layer(w, 0, "cuda")
    rng = np.random.default_rng(9)
    P, D = synth.PAGE_SIZE, 128
    L = int(d.seq_lens[0])
    npg = L // P
    kk = np.empty((npg * P, d.num_kv_heads, D), dtype=np.float32)
    for h in range(d.num_kv_heads):
        bs = int(d.block_size[h])
        nb = L // bs
        for ch in range(D):
            e = 2.0 ** -(4 + ch % 3)
            off = (ch % 5 - 2) * 3 * e
            j = rng.integers(0, 31, nb)
            j[0], j[1] = 0, 30
            vals = off + j * e / 2
            kk[:, h, ch] = np.repeat(vals, bs)[: npg * P]
    kb = torch.from_numpy(kk).to("cuda").to(torch.bfloat16)
    assert torch.equal(kb.float().cpu(), torch.from_numpy(kk))   # every key exact in bf16
    ids = d.page_table[0, :npg].long()
    d.k_pages[ids] = kb.view(npg, P, d.num_kv_heads, D).permute(0, 2, 1, 3)
    a = pipeline.DeviceLayer(d)
    b = pipeline.DeviceLayer(d)
    a.build_centroids()
    b.cent.codes.fill_(0xAB)
    b.build_centroids(fused=True)
    torch.cuda.synchronize()
    assert torch.equal(a.cent.codes, b.cent.codes)
    assert torch.equal(a.cent.scale.view(torch.int32), b.cent.scale.view(torch.int32))
    assert torch.equal(a.cent.zp, b.cent.zp)
    host = synth.host_layer(d)
    for h in range(d.num_kv_heads):
        bs = int(d.block_size[h])
        keys = O.gather_head_tokens(host.k_bits, host.page_table[0], L, h)
        want = O.quantize_centroids(O.build_centroids(keys, bs))
        n = want.codes.shape[0]
        got = O.unpack_codes(b.codes_of(0, h, n).cpu().numpy())
        assert np.array_equal(got, want.codes), h
        assert np.array_equal(want.scale, np.exp2(-(4 + np.arange(D) % 3)).astype(np.float32))
