"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Every case generates a seeded layer on the GPU, runs build + quantise,
score/select, sparse decode and the fused decode step, copies the touched
part of the layer to the host, and checks:
  codes / scales / zero points exact, selections exact up to counted
  boundary near-ties, outputs within max-abs 2e-2 / mean-abs 2e-3 of the
  oracle run on the GPU's own selection, and the fused step bit-identical to
  score/select followed by sparse decode.
"""

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


def _bits(t):
    return t.contiguous().view(torch.int16)


def run_case(lib, w, layer=0, seqs=None, modify=None, budget=None, data=None, fmt=0,
             flags=0, compare_out=True):
    abi, pipeline = lib
    d = data if data is not None else synth.make_layer(w, layer, "cuda")
    if modify is not None:
        modify(d)
    dl = pipeline.DeviceLayer(d, budget, fmt=fmt)
    bf16 = fmt == abi.ABSP_CENTROIDS_BF16
    dl.build_centroids()
    dl.score_select(flags=flags)
    dl.sparse_decode()
    dl.check()
    out_split = dl.out.clone()
    dl.out.zero_()
    dl.decode_step(flags=flags)
    dl.check()
    torch.cuda.synchronize()
    assert torch.equal(_bits(dl.out), _bits(out_split)), "fused step != select + decode"
    dl.out.zero_()
    dl.decode_step(flags=flags | abi.ABSP_STEP_EARLY_PREFETCH)
    dl.check()
    torch.cuda.synchronize()
    assert torch.equal(_bits(dl.out), _bits(out_split)), "early-prefetch step differs"

    S, Hkv = d.num_seqs, d.num_kv_heads
    seqs = list(range(S)) if seqs is None else list(seqs)
    hl = synth.host_layer(d, seqs)
    hl.budget = dl.budget
    sel = dl.sel.cpu().numpy()
    cnt = dl.sel_count.cpu().numpy()
    override = {(i, h): sel[s, h, :cnt[s, h]] for i, s in enumerate(seqs) for h in range(Hkv)}
    res = O.run_layer(hl, quantize="bf16" if bf16 else True, sel_override=override,
                      aggregate="max" if flags & abi.ABSP_STEP_GROUP_MAX else "sum")
    rep = PR.Report()
    for i, s in enumerate(seqs):
        for h in range(Hkv):
            hr = res.heads[(i, h)]
            rep.heads += 1
            n = hr.centroids.shape[0]
            if bf16:
                rows = dl.codes_of(s, h, n).cpu().numpy() if n else np.zeros((0, 256), np.uint8)
                PR.compare_bf16_centroids(rep, hr, rows)
            else:
                scale, zp = dl.params_of(s, h)
                packed = dl.codes_of(s, h, n).cpu().numpy() if n else np.zeros((0, 64), np.uint8)
                PR.compare_codes(rep, hr, packed, scale.cpu().numpy(), zp.cpu().numpy())
            PR.compare_selection(rep, hr, sel[s, h, :cnt[s, h]])
    outg = out_split[torch.as_tensor(seqs, device=out_split.device)].float().cpu().numpy()
    if compare_out:
        PR.compare_outputs(rep, outg, res.out)
    print(f"[parity] {w.name}: {rep.summary()}")
    assert rep.ok(), rep.notes[:10]
    return rep, dl, res


# ------------------------------------------------------------ small cases --

def test_tiny_8k(lib):
    run_case(lib, synth.WORKLOADS["tiny_8k"])


def test_ragged_lengths_two_heads(lib):
    w = synth.custom("ragged_small", 5, 8, 2, [1, 17, 100, 1000, 4097], [16, 64], 256, seed=11)
    run_case(lib, w)


def test_ragged_three_block_sizes(lib):
    w = synth.custom("ragged_3bs", 3, 12, 3, [3000, 64, 65], [16, 32, 64], 512, seed=12)
    run_case(lib, w)


def test_budget_covers_everything_is_dense(lib):
    w = synth.custom("select_all", 2, 8, 2, [700, 1500], [32, 16], 65536, seed=13)
    rep, dl, res = run_case(lib, w)
    cnt = dl.sel_count.cpu().numpy()
    assert cnt[0, 0] == 22 and cnt[1, 1] == 94


def test_single_block_and_empty_sequence(lib):
    w = synth.custom("tiny_seqs", 3, 4, 2, [5, 0, 16], [64, 16], 64, seed=14)
    rep, dl, res = run_case(lib, w)
    out = dl.out.float().cpu()
    assert torch.all(out[1] == 0)                       # empty sequence -> zeros
    assert dl.sel_count.cpu()[1].tolist() == [0, 0]


@pytest.mark.parametrize("hq,hkv", [(4, 4), (16, 2), (32, 2), (24, 3)])
def test_gqa_groups(lib, hq, hkv):
    bs = [16, 32, 64][:hkv] if hkv <= 3 else [16, 32, 64, 16]
    w = synth.custom(f"gqa{hq // hkv}", 2, hq, hkv, [2500, 1111], bs, 384, seed=15 + hq)
    run_case(lib, w)


def test_many_pairs_one_cta_each(lib):
    # 80 (sequence, KV head) pairs: the launch gives each pair one CTA (no
    # score exchange, no cluster merge); ragged lengths leave partial chunks
    # and partial lane groups
    lens = [1 + (977 * i) % 4100 for i in range(40)]
    w = synth.custom("many_pairs", 40, 8, 2, lens, [16, 64], 512, seed=41)
    run_case(lib, w)


@pytest.mark.parametrize("bs", [16, 64])
def test_uniform_block_size(lib, bs):
    w = synth.custom(f"uniform{bs}", 2, 16, 4, [5000, 3333], [bs] * 4, 1024, seed=20 + bs)
    run_case(lib, w)


def test_constant_channel_is_degenerate(lib):
    w = synth.custom("const_ch", 1, 8, 2, [2048], [16, 32], 256, seed=30)

    def modify(d):
        L = int(d.plan.seq_lens[0])
        ids = d.page_table[0, :L // 16].long()
        d.k_pages[ids, 0, :, 5] = 1.0
    rep, dl, res = run_case(lib, w, modify=modify)
    scale, zp = dl.params_of(0, 0)
    assert scale[5].item() == 0.0 and zp[5].item() == 0


def test_periodic_keys_resolve_ties_to_lower_index(lib):
    # keys repeat with a period of 4 blocks: only 4 distinct centroids, so
    # the K boundary falls inside a large group of exactly equal scores
    w = synth.custom("ties", 1, 8, 2, [4096], [16, 64], 400, seed=31, planted_blocks=0)

    def modify(d):
        for h, bs in enumerate(d.block_size.tolist()):
            ids = d.page_table[0, :256].long()
            k = d.k_pages[ids, h].reshape(-1, 128)            # [4096][128] logical
            per = 4 * bs
            k[:] = k[:per].repeat(4096 // per, 1)
            d.k_pages[ids, h] = k.view(256, 16, 128)
    rep, dl, res = run_case(lib, w, modify=modify)
    assert rep.near_ties == 0          # exact ties are resolved identically


def test_outlier_block_forces_radix_fallback(lib):
    # one block's keys scaled by 4096 stretch the score range so far that all
    # other scores share one histogram bin: the select falls back to radix
    w = synth.custom("outlier", 1, 8, 2, [32768], [16, 64], 1024, seed=32, planted_blocks=0)

    def modify(d):
        ids = d.page_table[0, 5:6].long()                 # block 5 of head 0 (bs 16)
        d.k_pages[ids, 0] = (d.k_pages[ids, 0].float() * 4096.0).to(torch.bfloat16)
    run_case(lib, w, modify=modify)


# ----------------------------------------------- BF16 centroid variant --

def _scale_kq(k_exp, q_exp):
    # powers of two: bf16 keys and queries stay exact, the codes do not move
    def modify(d):
        d.k_pages.mul_(2.0 ** k_exp)
        d.q.mul_(2.0 ** q_exp)
    return modify


def test_tiny_keys_far_below_one(lib):
    # score weights qbar * scale near 2^-60: the INT4 scoring's per-lane
    # working scale sits at its lower clamp
    run_case(lib, synth.custom("tiny_k_small", 2, 8, 2, [3000, 2300], [16, 64], 512, seed=81),
             modify=_scale_kq(-100, 40))


def test_tiny_keys_far_above_one(lib):
    # score weights near 2^80 (softmax logits near 2^80 make the attention
    # one-hot, so only codes and selection are compared)
    run_case(lib, synth.custom("tiny_k_large", 2, 8, 2, [3000, 2300], [16, 32], 512, seed=82),
             modify=_scale_kq(50, 30), compare_out=False)


def test_bf16_centroids_tiny(lib):
    abi, _ = lib
    run_case(lib, synth.WORKLOADS["tiny_8k"], fmt=abi.ABSP_CENTROIDS_BF16)


def test_bf16_centroids_ragged_gqa16(lib):
    abi, _ = lib
    w = synth.custom("bf16_ragged", 3, 32, 2, [3000, 77, 1025], [32, 16], 384, seed=60)
    run_case(lib, w, fmt=abi.ABSP_CENTROIDS_BF16)


def test_bf16_centroids_llama31_8b_32k(lib):
    abi, _ = lib
    run_case(lib, synth.WORKLOADS["llama31_8b_32k"], fmt=abi.ABSP_CENTROIDS_BF16)


# ------------------------------------------- group-max aggregation variant --

@pytest.mark.parametrize("fmt", [0, 1])
def test_group_max_tiny(lib, fmt):
    abi, _ = lib
    run_case(lib, synth.WORKLOADS["tiny_8k"], fmt=fmt, flags=abi.ABSP_STEP_GROUP_MAX)


def test_group_max_ragged_gqa16(lib):
    abi, _ = lib
    w = synth.custom("gmax_ragged", 3, 32, 2, [3000, 77, 1025], [32, 16], 384, seed=61)
    run_case(lib, w, flags=abi.ABSP_STEP_GROUP_MAX)


def test_group_max_llama31_8b_32k(lib):
    abi, _ = lib
    run_case(lib, synth.WORKLOADS["llama31_8b_32k"], flags=abi.ABSP_STEP_GROUP_MAX)


@pytest.mark.parametrize("wname", ["tiny_8k", "llama31_8b_32k"])
def test_throughput_hint_matches_the_oracle(lib, wname):
    # ABSP_STEP_THROUGHPUT halves the CTAs per head: the same selection, the
    # output equal up to the merge order's rounding, so within the oracle
    # tolerance and bf16-close to the default step's
    abi, pipeline = lib
    rep, dl, res = run_case(lib, synth.WORKLOADS[wname])
    want = dl.out.clone()
    dl.out.zero_()
    dl.decode_step(flags=abi.ABSP_STEP_THROUGHPUT | abi.ABSP_STEP_EARLY_PREFETCH)
    dl.check()
    torch.cuda.synchronize()
    got = dl.out.float().cpu().numpy()
    rep2 = PR.Report()
    PR.compare_outputs(rep2, got, res.out)
    assert rep2.ok(), rep2.notes[:10]
    diff = (dl.out.float() - want.float()).abs().max().item()
    assert diff <= 2e-2 * max(1.0, want.float().abs().max().item()), diff


def test_host_buffers_match_device_step(lib):
    abi, pipeline = lib
    w = synth.custom("host_io", 2, 8, 2, [3000, 900], [16, 64], 512, seed=40)
    d = synth.make_layer(w, 0, "cuda")
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    dl.decode_step()
    torch.cuda.synchronize()
    # pinned (device-mapped: the kernel reads and writes them directly) and
    # pageable host buffers (copied through the workspace) give the same
    for pin in (True, False):
        for flags in (0, abi.ABSP_STEP_EARLY_PREFETCH):
            q_host = d.q.cpu()
            out_host = torch.zeros_like(q_host)
            if pin:
                q_host, out_host = q_host.pin_memory(), out_host.pin_memory()
            dl.decode_step_host(q_host, out_host, flags=flags)
            torch.cuda.synchronize()
            dl.check()
            assert torch.equal(_bits(out_host), _bits(dl.out.cpu())), (pin, flags)


def test_repeated_steps_are_deterministic(lib):
    abi, pipeline = lib
    d = synth.make_layer(synth.WORKLOADS["tiny_8k"], 0, "cuda")
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    dl.decode_step()
    a = dl.out.clone()
    for _ in range(3):
        dl.decode_step()
    torch.cuda.synchronize()
    assert torch.equal(_bits(a), _bits(dl.out))


def test_concurrent_host_threads(lib):
    # the library's launch path (per-device caches, attribute set-up) driven
    # from several host threads at once, each with its own stream and layer;
    # every thread's results equal a serial run bit for bit
    import threading
    abi, pipeline = lib
    ws = [synth.custom(f"mt{i}", 1, 8 * (1 + i % 2), 2, [3000 + 700 * i], [16, 64], 512,
                       seed=300 + i) for i in range(4)]
    layers, want, streams = [], [], []
    for w in ws:
        d = synth.make_layer(w, 0, "cuda")
        streams.append(torch.cuda.Stream())
        dl = pipeline.DeviceLayer(d, stream=streams[-1].cuda_stream)
        dl.build_centroids()
        torch.cuda.synchronize()
        layers.append(dl)
    for dl in layers:
        dl.decode_step(flags=abi.ABSP_STEP_EARLY_PREFETCH)
        torch.cuda.synchronize()
        want.append(dl.out.clone())
    errors = []

    def work(dl):
        try:
            for i in range(25):
                dl.decode_step(flags=abi.ABSP_STEP_EARLY_PREFETCH if i % 2 else 0)
                dl.score_select()
                dl.sparse_decode()
        except Exception as e:  # reported by the main thread
            errors.append(e)

    ts = [threading.Thread(target=work, args=(dl,)) for dl in layers]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    torch.cuda.synchronize()
    assert not errors, errors
    for dl, w in zip(layers, want):
        dl.check()
        assert torch.equal(_bits(dl.out), _bits(w))


# ----------------------------------------------------- device-side faults --

def _fault_layer(lib):
    abi, pipeline = lib
    w = synth.custom("faults", 2, 8, 2, [1000, 600], [16, 32], 256, seed=50)
    d = synth.make_layer(w, 0, "cuda")
    return abi, pipeline, d


def test_page_id_out_of_range_is_reported(lib):
    abi, pipeline, d = _fault_layer(lib)
    dl = pipeline.DeviceLayer(d)
    d.page_table[1, 3] = d.k_pages.shape[0] + 5      # bad physical page
    with pytest.raises(abi.AbspError) as e:
        dl.build_centroids()
    assert e.value.status == abi.ABSP_ERR_DEVICE_FAULT
    dl.decode_step()
    st, detail = abi.absp_check_device_error(dl.ws)
    # the attention may or may not select the bad page; the call must not
    # fault the context either way
    assert st in (abi.ABSP_OK, abi.ABSP_ERR_DEVICE_FAULT)
    torch.cuda.synchronize()


def test_sequence_length_beyond_page_table_is_reported(lib):
    abi, pipeline, d = _fault_layer(lib)
    dl = pipeline.DeviceLayer(d)
    d.seq_lens[0] = d.page_table.shape[1] * 16 + 1
    with pytest.raises(abi.AbspError) as e:
        dl.build_centroids()
    assert e.value.status == abi.ABSP_ERR_DEVICE_FAULT
    dl.decode_step()
    st, _ = abi.absp_check_device_error(dl.ws)
    assert st == abi.ABSP_ERR_DEVICE_FAULT


def test_selected_block_out_of_range_is_reported(lib):
    abi, pipeline, d = _fault_layer(lib)
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    dl.score_select()
    dl.check()
    dl.sel[0, 1, 0] = 10_000
    dl.sparse_decode()
    st, detail = abi.absp_check_device_error(dl.ws)
    assert st == abi.ABSP_ERR_DEVICE_FAULT and detail == 0
    dl.sel_count[1, 0] = dl.kmax + 1
    dl.sparse_decode()
    st, detail = abi.absp_check_device_error(dl.ws)
    assert st == abi.ABSP_ERR_DEVICE_FAULT
    dl.score_select()
    dl.sparse_decode()
    dl.check()                                       # clean again


# ------------------------------------------------------ named workloads --

def test_llama31_8b_32k_full(lib):
    rep, dl, res = run_case(lib, synth.WORKLOADS["llama31_8b_32k"])


def test_llama31_8b_32k_planted_recall(lib):
    # method diagnostic: every planted span is selected by the GPU
    abi, pipeline = lib
    w = synth.WORKLOADS["llama31_8b_32k"]
    d = synth.make_layer(w, 0, "cuda")
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    dl.score_select()
    sel = dl.sel.cpu().numpy()
    cnt = dl.sel_count.cpu().numpy()
    for h, bs in enumerate(d.block_size.tolist()):
        got = set(sel[0, h, :cnt[0, h]].tolist())
        for st in d.plan.planted[0][h]:
            assert set(range(int(st) // bs, (int(st) + 64) // bs)) <= got


@pytest.mark.parametrize("layer", [0, 35])
def test_qwen3_8b_128k_layer(lib, layer):
    run_case(lib, synth.WORKLOADS["qwen3_8b_128k_36l"], layer=layer)


def test_max_blocks_per_head(lib):
    # 262144 tokens at block size 16: head 0 holds ABSP_MAX_BLOCKS_PER_HEAD
    # (16384) code rows, the largest score buffer and selection bitmap
    abi, _ = lib
    w = synth.custom("max_blocks", 1, 8, 2, [262144], [16, 64], 4096, seed=51)
    rep, dl, res = run_case(lib, w)
    assert res.heads[(0, 0)].centroids.shape[0] == 16384


def test_max_budget(lib):
    # the largest token budget (65536) over a 131072-token context: half of
    # every head's blocks are selected, 32 pages per warp, the longest list
    w = synth.custom("max_budget", 1, 8, 2, [131072], [16, 64], 65536, seed=52)
    rep, dl, res = run_case(lib, w)
    cnt = dl.sel_count.cpu().numpy()
    assert cnt[0].tolist() == [4096, 1024]


def test_batch32_32k_sampled(lib):
    run_case(lib, synth.WORKLOADS["batch32_32k_8l"], layer=3, seqs=[0, 17, 31])


def test_ragged64_paged_sampled(lib):
    w = synth.WORKLOADS["ragged64_paged"]
    lens = synth.draw_seq_lens(w)
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, 33})
    run_case(lib, w, seqs=seqs)


def test_rebuild_8x128k_sampled(lib):
    run_case(lib, synth.WORKLOADS["rebuild_8x128k"], seqs=[0, 7])
