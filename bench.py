#!/usr/bin/env python
"""Decode benchmark: sparse-attention layer-steps/s at 32K context on B200.

Workload: a Llama-3.1-8B-shaped attention layer (32 query / 8 KV heads,
head_dim 128, batch 1, 32768-token paged bf16 cache, block sizes per KV head
drawn from {16, 32, 64} with probabilities {0.25, 0.25, 0.5}, token budget
2048, INT4 centroids).  One benchmark step decodes one token through
`--layers` (default 64) such layers, each with its own cache, centroids and
query, so the working set (8 GiB) is far larger than L2.  Each layer-step is
one absp_decode_step_ex launch with ABSP_STEP_EARLY_PREFETCH; the
layer-steps of a step are captured in a CUDA graph.  Every launch waits for
the previous one to finish before it reads its query, as consecutive layers
of a real decode would; what overlaps the previous launch is only the
launch itself and the reads of this layer's cache-side data (lengths, page
table, centroid codes, per-channel parameters), which no decode kernel
writes.  `variants.plain` is the same measurement with absp_decode_step
(nothing read before the previous launch completed).

value   = layer-steps/s over all ranks (weak scaling: every rank decodes its
          own layer stack, no collective on the data path);
e2e     = the same through absp_decode_step_host_ex (same flags) with
          pinned host buffers (the kernel reads each layer's query from host
          memory and writes its output there, inside every layer-step);
roofline= algorithmic bytes of a layer-step (centroid codes + per-channel
          parameters + valid selected K/V rows + q and out) / average launch
          time, against the measured HBM copy bandwidth;
rebuild = centroid build + INT4 quantisation of every layer (steps 1-2),
          timed separately (it runs once per cache, not per token); the
          oracle's steps 1-2 are timed under cpu_baseline.rebuild;
calibration = per-head normalised recall at block sizes 16/32/64 on a set of
          heads of varied concentration, and the block-size allocation it
          gives at the centroid memory of a uniform block size 32.

`--impl reference` times the CPU oracle on the same workload instead.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode layer-steps/s at 32K ctx; achieved HBM GB/s vs B200 peak"
UNIT = "layer-steps/s"
WORKLOAD = "llama31_8b_32k"
WORKLOAD_DESC = (f"{WORKLOAD}: Llama-3.1-8B-shaped attention layer decode, 32 q / 8 kv "
                 f"heads, head_dim 128, batch 1, ctx 32768, budget 2048 tokens, "
                 f"block sizes per kv head from {{16,32,64}}, INT4 centroids")
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
KERNEL_SOURCES = [os.path.join(ROOT, "block_sparse_attention_kv_b200", "csrc", f)
                  for f in ("decode.cu", "absp_internal.cuh")]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="absp", choices=["absp", "reference"])
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the long-context and batched workloads (reported "
                         "under 'workloads')")
    return ap.parse_args()


# ------------------------------------------------------------- helpers --

class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting"}

    def __init__(self, index: int, period: float = 0.005):
        super().__init__(daemon=True)
        self.index, self.period = index, period
        self.sm, self.reasons, self.max_mhz = [], set(), None
        self._halt = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def run(self):
        if not self.ok:
            return
        nv = self.nv
        while not self._halt.is_set():
            try:
                self.sm.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)
        if not self.sm:
            return None
        return {"sm_mhz": float(statistics.median(self.sm)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.sm), "reasons": sorted(self.reasons)}


SLOW_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(clocks) -> list:
    """Why a timed region's clock record disqualifies it (empty: it stands).

    A hardware or thermal slowdown seen during the region, or a median SM
    clock well below the maximum with no reason reported (a clock lock left
    behind by another process).  A software power cap is kept.
    """
    if not clocks:
        return []
    why = [r for r in clocks.get("reasons", []) if r in SLOW_REASONS]
    mx = clocks.get("sm_max_mhz")
    if not why and mx and clocks["sm_mhz"] < 0.85 * mx and \
            "sw_power_cap" not in clocks.get("reasons", []):
        why.append("sm clock below 85 % of max with no reason")
    return why


def timed_with_clocks(timed, make_sampler, dist=None, device=None):
    """One timed region with its clock record, timed once more when the
    record disqualifies it on any rank.

    `timed()` returns the region's max-over-ranks milliseconds; every rank
    takes the same collective steps, since whether to time again is itself
    a max over ranks.  Returns (ms, clocks); a second measurement's clocks
    carry the first under "remeasured_after".
    """
    sampler = make_sampler()
    sampler.start()
    ms = timed()
    clocks = sampler.stop()
    why = clocks_rejected(clocks)
    if reduce_max(1.0 if why else 0.0, dist, device) > 0:
        first = {"ms": ms, "why": why, "clocks": clocks}
        sampler = make_sampler()
        sampler.start()
        ms = timed()
        clocks = sampler.stop()
        if clocks is not None:
            clocks["remeasured_after"] = first
    return ms, clocks


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_text(src: str) -> str:
    """C/C++/CUDA source without its comments and blank space.

    Comments go (a block comment counts as one space) except inside string
    and character literals, runs of spaces and tabs become one space (inside
    literals too), and blank lines go; line breaks between code stay, since
    a preprocessor directive ends at one.
    """
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == "/" and src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif c == "/" and src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c and src[j] != "\n":
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = (" ".join(l.split()) for l in "".join(out).split("\n"))
    return "\n".join(l for l in lines if l)


def kernel_source_hash() -> str:
    """sha256 (16 hex digits) of the decode kernel's code, comments ignored."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, encoding="utf-8") as f:
            h.update(code_text(f.read()).encode())
        h.update(b"\0")
    return h.hexdigest()[:16]


def recorded_traffic():
    """ncu DRAM bytes per launch, if recorded for the current kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        if rec.get("source_sha") == kernel_source_hash():
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def step_bytes(d, sel, cnt, block_size=None, bf16=False):
    """Algorithmic bytes of one decode layer-step of layer data `d`."""
    lens = d.seq_lens.cpu().numpy()
    S, Hkv, Hq = d.num_seqs, d.num_kv_heads, d.num_q_heads
    bsz = d.block_size if block_size is None else block_size
    total = S * Hq * 128 * 2 * 2                       # q in + out
    for s in range(S):
        L = int(lens[s])
        for h in range(Hkv):
            bs = int(bsz[h])
            n = (L + bs - 1) // bs
            total += n * 256 if bf16 else n * 64 + 128 * 8   # centroid rows (+ scale/zp)
            toks = 0
            for b in sel[s, h, :cnt[s, h]]:
                toks += min(bs, L - int(b) * bs)
            total += toks * 2 * 128 * 2                # K and V rows
    return total


def rebuild_bytes(d):
    lens = d.seq_lens.cpu().numpy()
    tot = 0
    for s in range(d.num_seqs):
        L = int(lens[s])
        for h in range(d.num_kv_heads):
            bs = int(d.block_size[h])
            tot += L * 256 + ((L + bs - 1) // bs) * 64 + 128 * 8
    return tot


# ---------------------------------------------------------------- ranks --

def bench_config(layers: int, world: int) -> dict:
    """The workload description both arms report."""
    return {
        "workload": WORKLOAD_DESC,
        "layers_per_step": layers,
        "step": f"one decode token through {layers} layers with distinct caches",
        "l2": f"inputs larger than L2: {layers} distinct layer caches (~{layers * 128 // 1024} GiB)",
        "parallelism": f"dp{world} (independent layer stacks per GPU)",
    }


def rank_layer_ids(rank: int, layers: int) -> list:
    """Layer seeds of one rank: every rank decodes its own layer stack."""
    return [rank * layers + i for i in range(layers)]


def reduce_max(value: float, dist=None, device=None) -> float:
    """Max over ranks (identity on one process)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, layers: int, steps: int, ms: float) -> float:
    """Whole-job layer-steps/s: all ranks' layer-steps over the max time."""
    return world * layers * steps / (ms / 1e3)


def rebuild_large(dev, stream, abi, pipeline, synth):
    """Steps 1-2 at batch 8 x 131072 tokens (8 KV heads, mixed block sizes)."""
    w = synth.WORKLOADS["rebuild_8x128k"]
    with torch.cuda.stream(stream):
        d = synth.make_layer(w, 0, dev)
        y = pipeline.DeviceLayer(d, stream=stream.cuda_stream)
    ws = abi.alloc_workspace(abi.absp_build_workspace_size(y.kv), dev)
    sc = stream.cuda_stream
    for _ in range(2):
        abi.absp_build_quantize_centroids(y.kv, ws, y.cent, sc)
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = 5
    e0.record(stream)
    for _ in range(reps):
        abi.absp_build_quantize_centroids(y.kv, ws, y.cent, sc)
    e1.record(stream)
    stream.synchronize()
    st, _ = abi.absp_check_device_error(ws, sc)
    assert st == abi.ABSP_OK
    ms = e0.elapsed_time(e1) / reps
    nbytes = rebuild_bytes(d)
    del y, d, ws
    torch.cuda.empty_cache()
    return {"workload": "rebuild_8x128k: 8 sequences x 131072 tokens, 8 KV heads",
            "ms": ms, "bytes": nbytes, "achieved_gbs": nbytes / (ms * 1e-3) / 1e9}


# The other workloads, each at the layer count it is stated with; a timed
# graph replays every layer once per step, so the layer-steps of one replay
# read far more than L2 holds (selected K/V + codes per replay: Qwen3 128K
# 36 x ~19 MB, batch 32 8 x ~144 MB, ragged 64 2 x ~0.6 GB, GQA 16 4 x
# ~0.1 GB).  The ragged batch is one layer of 64 sequences; two distinct
# caches keep a replay from finding the previous one in L2.
OTHER_WORKLOADS = (("qwen3_8b_128k_36l", 36), ("batch32_32k_8l", 8), ("ragged64_paged", 2),
                   ("gqa16_batch96_16k", 4))


def other_workloads(dev, stream, abi, pipeline, synth, timed, steps, warmup, peak,
                    parity: bool = True):
    """The fused early-prefetch step on the long-context and batched
    workloads: per layer-step time and algorithmic bytes, same method as the
    headline (CUDA graph over distinct layer caches, CUDA events), and a
    parity record of the oracle on one of the timed layers (two sequences of
    a batch)."""
    out = {}
    sc = stream.cuda_stream
    flags = abi.ABSP_STEP_EARLY_PREFETCH
    for name, nl in OTHER_WORKLOADS:
        w = synth.WORKLOADS[name]
        ys, nb = [], []
        t_gen = time.perf_counter()
        with torch.cuda.stream(stream):
            for i in range(nl):
                y = pipeline.DeviceLayer(synth.make_layer(w, i, dev), stream=sc)
                y.build_centroids()
                y.score_select()
                stream.synchronize()
                nb.append(step_bytes(y.data, y.sel.cpu().numpy(), y.sel_count.cpu().numpy()))
                abi.absp_decode_step_ex(y.kv, y.cent, y.data.q, y.budget, y.out, y.ws,
                                        flags, sc)
                ys.append(y)
        stream.synchronize()
        t_gen = time.perf_counter() - t_gen
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for y in ys:
                abi.absp_decode_step_ex(y.kv, y.cent, y.data.q, y.budget, y.out, y.ws,
                                        flags, sc)
        with torch.cuda.stream(stream):
            ms = timed(g, steps, warmup)
        for y in ys:
            y.check()
        us = ms / (steps * nl) * 1e3
        bpl = float(np.mean(nb))
        gbs = bpl / (us * 1e-6) / 1e9
        rec = {"us_per_layer_step": us, "layers": nl, "bytes_per_launch": bpl,
               "achieved_gbs": gbs, "frac": gbs / peak, "value": 1e6 / us,
               "unit": UNIT, "sequences": w.num_seqs, "kv_heads": w.num_kv_heads,
               "q_heads": w.num_q_heads, "budget": w.budget,
               "ctx": w.ctx if w.ragged is None else f"log-uniform {list(w.ragged)}",
               "setup_s": t_gen}
        if parity:
            S = ys[0].data.num_seqs
            seqs = [0] if S == 1 else [0, S - 1]
            rec["parity"] = parity_record(ys[0], name, seqs)
        out[name] = rec
        del g, ys
        torch.cuda.empty_cache()
    return out


PIPELINE_STREAMS = 8


def pipelined_variant(layers, stream, abi, timed, steps, warmup):
    """The same early-prefetch launches as the headline graph, spread
    round-robin over PIPELINE_STREAMS streams inside one graph, so that
    independent layer-steps overlap: a throughput mode for work without a
    layer-to-layer dependency, not a decode order.  Returns the graph's
    milliseconds over `steps` replays.  The launches carry the throughput
    hint (half as many CTAs per head, so that more launches are resident)."""
    flags = abi.ABSP_STEP_EARLY_PREFETCH | abi.ABSP_STEP_THROUGHPUT
    side = [torch.cuda.Stream(device=stream.device) for _ in range(PIPELINE_STREAMS)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for sd in side:                      # fork from the capturing stream
            sd.wait_stream(stream)
        for i, x in enumerate(layers):
            sd = side[i % PIPELINE_STREAMS]
            abi.absp_decode_step_ex(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, flags,
                                    sd.cuda_stream)
        for sd in side:                      # join back before the capture ends
            stream.wait_stream(sd)
    with torch.cuda.stream(stream):
        ms = timed(g, steps, warmup)
    for x in layers:
        x.check()
    del g
    return ms


# ------------------------------------------------------- CPU oracle leg --

def oracle_layer_sample(layer_index: int = 0, heads=None):
    """Host copy of one layer plus the oracle's prebuilt centroids (of the
    KV heads in `heads`, all when None)."""
    from block_sparse_attention_kv_b200 import synth
    w = synth.WORKLOADS[WORKLOAD]
    d = synth.make_layer(w, layer_index, "cpu")
    return _oracle_prep(synth.host_layer(d), heads)


def _oracle_prep(hl, heads=None):
    """(units, G, budget) of a host layer: one unit per (sequence, KV head),
    each with the oracle's prebuilt dequantised centroids."""
    from oracle import absp_oracle as O
    prep = []
    for s in range(hl.q_bits.shape[0]):
        qf = O.decode_bf16(hl.q_bits[s])
        for h in range(len(hl.block_size)):
            if heads is not None and h not in heads:
                continue
            keys, vals = O.head_keys_values(hl, s, h)
            bs = int(hl.block_size[h])
            chat = O.dequantize(O.quantize_centroids(O.build_centroids(keys, bs)))
            prep.append((qf, h, chat, keys, vals, bs, int(hl.seq_lens[s])))
    G = hl.q_bits.shape[1] // len(hl.block_size)
    return prep, G, int(hl.budget)


def sample_lengths(lens, k: int) -> list:
    """k lengths evenly spaced through the sorted `lens` (the midpoints of k
    equal slices of the sorted list)."""
    lens = np.sort(np.asarray(lens))
    k = min(k, len(lens))
    return [int(lens[(2 * i + 1) * len(lens) // (2 * k)]) for i in range(k)]


def oracle_workload_sample(name: str, k: int = 4):
    """A bounded host sample of workload `name` for the oracle: k of its
    sequences (evenly spaced in its sorted length list, so a ragged batch is
    covered from short to long), generated as a small layer with the same
    head counts, block sizes and budget.  Returns (prep, G, budget, lengths,
    units per layer-step of the whole workload)."""
    from block_sparse_attention_kv_b200 import synth
    w = synth.WORKLOADS[name]
    pick = sample_lengths(synth.draw_seq_lens(w), k)
    k = len(pick)
    bs = [int(b) for b in synth.draw_block_sizes(w, 0)]
    sw = synth.custom(f"{name}_sample", k, w.num_q_heads, w.num_kv_heads, pick, bs,
                      w.budget, seed=w.seed)
    prep, G, budget = _oracle_prep(synth.host_layer(synth.make_layer(sw, 0, "cpu")))
    return prep, G, budget, pick, w.num_seqs * w.num_kv_heads


def oracle_workloads(seconds: float) -> dict:
    """The oracle's steps 3-5 on a bounded sample of each of the other
    workloads, 1 thread, about `seconds` each; the layer-step time is the
    mean time of a sampled (sequence, KV head) unit times the workload's
    units per layer-step."""
    out = {}
    for name, _ in OTHER_WORKLOADS:
        prep, G, budget, pick, units = oracle_workload_sample(name)
        time_oracle(prep, G, budget, steps=1)                    # warm
        done, el = time_oracle(prep, G, budget, seconds=seconds)
        ms = el / done * units * 1e3
        out[name] = {"value": 1e3 / ms, "unit": UNIT, "ms_per_layer_step": ms, "cores": 1,
                     "kind": "oracle",
                     "sample": f"{done} (sequence, KV head) units of {len(pick)} sequences "
                               f"(lengths {pick}) generated with the workload's head counts, "
                               f"block sizes and budget; mean unit time x {units} units "
                               f"per layer-step; numpy fp64, 1 thread, {el:.1f} s"}
    return out


def time_oracle(prep, G, budget, steps: int = None, seconds: float = None):
    """Runs oracle decode (steps 3-5) over (seq, head) units; returns
    (units done, elapsed s)."""
    from oracle import absp_oracle as O
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(limits=1)
    except Exception:
        lim = None
    t0 = time.perf_counter()
    done = 0
    while True:
        if steps is not None and done >= steps:
            break
        if seconds is not None and time.perf_counter() - t0 >= seconds:
            break
        qf, h, chat, keys, vals, bs, L = prep[done % len(prep)]
        O.decode_head(qf, h, G, chat, keys, vals, bs, L, budget)
        done += 1
    el = time.perf_counter() - t0
    if lim is not None:
        lim.unregister() if hasattr(lim, "unregister") else None
    return done, el


def time_oracle_rebuild(seconds: float):
    """The oracle's steps 1-2 (centroids + INT4 codes) per KV head of the
    workload's layer 0, 1 thread, for about `seconds`; returns (ms per layer
    of Hkv heads, heads done)."""
    from block_sparse_attention_kv_b200 import synth
    from oracle import absp_oracle as O
    w = synth.WORKLOADS[WORKLOAD]
    hl = synth.host_layer(synth.make_layer(w, 0, "cpu"))
    heads = [(O.head_keys_values(hl, 0, h)[0], int(hl.block_size[h]))
             for h in range(len(hl.block_size))]
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(limits=1)
    except Exception:
        lim = None
    t0 = time.perf_counter()
    done = 0
    while done == 0 or time.perf_counter() - t0 < seconds:
        keys, bs = heads[done % len(heads)]
        O.quantize_centroids(O.build_centroids(keys, bs))
        done += 1
    el = time.perf_counter() - t0
    if lim is not None and hasattr(lim, "unregister"):
        lim.unregister()
    return el / done * len(heads) * 1e3, done


def _oracle_worker(task):
    """One process of the all-cores oracle timing: (units done, seconds)."""
    seconds, head, barrier = task
    prep, G, budget = oracle_layer_sample(0, heads=[head])
    # every worker times the same window; a worker that never arrives
    # breaks the barrier for the others instead of holding them forever
    barrier.wait(timeout=300)
    return time_oracle(prep, G, budget, seconds=seconds)


def time_oracle_all_cores(seconds: float, max_procs: int = 32):
    """The oracle on one process per host core (at most max_procs), each on
    one KV head of the workload's layer 0; spawn start, so it is safe after
    the GPU was used.  Returns (layer-steps/s, processes, units, seconds)."""
    import multiprocessing as mp
    n = max(1, min(os.cpu_count() or 1, max_procs))
    ctx = mp.get_context("spawn")
    nh = synth_kv_heads()
    with ctx.Manager() as mgr:
        bar = mgr.Barrier(n)
        with ctx.Pool(n) as pool:
            res = pool.map(_oracle_worker, [(seconds, i % nh, bar) for i in range(n)])
    units = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    return (units / nh) / el, n, units, el


def synth_kv_heads() -> int:
    from block_sparse_attention_kv_b200 import synth
    return synth.WORKLOADS[WORKLOAD].num_kv_heads


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    prep, G, budget = oracle_layer_sample(0)
    units_per_layer_step = len(prep)
    time_oracle(prep, G, budget, steps=args.warmup)
    done, el = time_oracle(prep, G, budget, steps=args.steps)
    layer_steps = done / units_per_layer_step
    value = layer_steps / el
    sample = (f"{args.steps} steps, each the oracle's steps 3-5 (score, top-K, "
              f"attention) for one (sequence, KV head) of a {WORKLOAD} layer "
              f"(1/{units_per_layer_step} layer-step), numpy fp64, 1 thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / max(done, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(args.layers, args.gpus),
            "launch": "the CPU oracle (numpy fp64), one host thread, rank 0 only; each step "
                      "one (sequence, KV head) unit of a layer-step",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    if not args.no_workloads:
        line["workloads"] = oracle_workloads(min(3.0, args.cpu_seconds))
    print(json.dumps(line), flush=True)


# ------------------------------------------------ block-size calibration --

def calibration_summary(dev, synth):
    """Per-head sensitivity on the 8-head calibration set and the block-size
    allocation it gives at the centroid memory of a uniform block size 32."""
    from block_sparse_attention_kv_b200 import calibrate as cal
    w = synth.WORKLOADS["calib_8h_32k"]
    d = synth.make_layer(w, 0, dev)
    t0 = time.perf_counter()
    c = cal.calibrate(d, lambda s, h: synth.planted_mask(d.plan, s, h))
    budget = int(c.rows[:, 1].sum())
    choice, _, used = cal.allocate(c.normalised, c.rows, budget)
    ms = (time.perf_counter() - t0) * 1e3
    rec = c.recall
    H = rec.shape[0]
    del d
    return {
        "workload": "calib_8h_32k: 8 KV heads (32 q), 32K ctx, budget 2048, 512 planted "
                    "q-aligned tokens per head in spans of 4 .. 512 tokens",
        "span_tokens": [int(x) for x in w.planted_lens],
        "block_sizes": list(c.block_sizes),
        "normalised_recall": [[round(float(v), 4) for v in row] for row in c.normalised],
        "recall_uniform": {str(bs): float(rec[:, j].mean()) for j, bs in enumerate(c.block_sizes)},
        "alloc_budget_rows": budget,
        "alloc_rows": int(used),
        "alloc_block_sizes": [int(c.block_sizes[j]) for j in choice],
        "recall_alloc": float(np.mean([rec[h, choice[h]] for h in range(H)])),
        "ms": ms,
    }


# ------------------------------------------------------ parity record --

def parity_record(x, name: str, seqs=None) -> dict:
    """The oracle against the library on one layer that the timed region
    decoded, checked after it: INT4 codes, scales and zero points exact,
    selections exact up to counted boundary near-ties, and the output that
    the timed launches left in x.out within the tolerances of the oracle
    run on the library's own selection, for every KV head of the sampled
    sequences."""
    from block_sparse_attention_kv_b200 import synth
    from oracle import absp_oracle as O
    from oracle import parity as PR
    d = x.data
    S, Hkv = d.num_seqs, d.num_kv_heads
    seqs = list(range(S)) if seqs is None else list(seqs)
    t0 = time.perf_counter()
    x.score_select()                  # the selection the fused launches made
    torch.cuda.synchronize()
    x.check()
    hl = synth.host_layer(d, seqs)
    hl.budget = x.budget
    sel = x.sel.cpu().numpy()
    cnt = x.sel_count.cpu().numpy()
    over = {(i, h): sel[s, h, :cnt[s, h]] for i, s in enumerate(seqs) for h in range(Hkv)}
    res = O.run_layer(hl, sel_override=over)
    rep = PR.Report()
    for i, s in enumerate(seqs):
        for h in range(Hkv):
            hr = res.heads[(i, h)]
            rep.heads += 1
            n = hr.centroids.shape[0]
            scale, zp = x.params_of(s, h)
            PR.compare_codes(rep, hr, x.codes_of(s, h, n).cpu().numpy(),
                             scale.cpu().numpy(), zp.cpu().numpy())
            PR.compare_selection(rep, hr, sel[s, h, :cnt[s, h]])
    out = x.out[torch.as_tensor(seqs, device=x.out.device)].float().cpu().numpy()
    PR.compare_outputs(rep, out, res.out)
    return {"workload": name, "sequences": seqs, "kv_heads": rep.heads,
            "code_mismatch": rep.code_mismatch, "param_mismatch": rep.param_mismatch,
            "sel_mismatch": rep.sel_mismatch, "near_ties": rep.near_ties,
            "out_max_abs": rep.out_max_abs, "out_mean_abs": rep.out_mean_abs,
            "tolerance": {"out_max_abs": PR.OUT_MAX_ABS, "out_mean_abs": PR.OUT_MEAN_ABS,
                          "tie_rel": PR.TIE_REL},
            "ok": rep.ok(), "seconds": time.perf_counter() - t0}


# ----------------------------------------------------------- GPU arm --

def gpu_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from block_sparse_attention_kv_b200 import build as absp_build
    if rank == 0 or world == 1:
        absp_build.build()
    if dist is not None:
        dist.barrier()
    from block_sparse_attention_kv_b200 import abi, pipeline, synth

    w = synth.WORKLOADS[WORKLOAD]
    L = args.layers
    stream = torch.cuda.Stream(device=dev)
    layers = []
    with torch.cuda.stream(stream):
        for i in rank_layer_ids(rank, L):
            d = synth.make_layer(w, i, dev)
            layers.append(pipeline.DeviceLayer(d, stream=stream.cuda_stream))
    stream.synchronize()

    # steps 1-2 for every layer, timed (once per cache): the one-call build
    # (absp_build_quantize_centroids, one fused launch per layer here), and
    # the two separate calls
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ws_n = max(abi.absp_build_workspace_size(x.kv) for x in layers)
    bws = abi.alloc_workspace(ws_n, dev)
    sc = stream.cuda_stream

    def time_builds(fused: bool) -> float:
        def one(x):
            if fused:
                abi.absp_build_quantize_centroids(x.kv, bws, x.cent, sc)
            else:
                abi.absp_build_centroids(x.kv, bws, sc)
                abi.absp_quantize_centroids(x.kv, bws, x.cent, sc)
        for x in layers[:2]:                           # warm-up
            one(x)
        stream.synchronize()
        ev0.record(stream)
        for x in layers:
            one(x)
        ev1.record(stream)
        stream.synchronize()
        st, _ = abi.absp_check_device_error(bws, sc)
        assert st == abi.ABSP_OK, "device fault while building centroids"
        return ev0.elapsed_time(ev1) / L

    rebuild_two_ms = time_builds(False)
    rebuild_ms = time_builds(True)
    rb_bytes = sum(rebuild_bytes(x.data) for x in layers) / L
    del bws
    rb_large = None if args.no_variants else rebuild_large(dev, stream, abi, pipeline, synth)
    calib = None if args.no_variants or rank != 0 else calibration_summary(dev, synth)

    # algorithmic bytes from each layer's own selection
    nbytes = []
    for x in layers:
        x.score_select()
        stream.synchronize()
        nbytes.append(step_bytes(x.data, x.sel.cpu().numpy(), x.sel_count.cpu().numpy()))
        x.decode_step()                                # warm: attributes, occupancy
    stream.synchronize()
    for x in layers:
        x.check()
    bytes_per_launch = float(np.mean(nbytes))

    # CUDA graph of one step = L layer-steps
    EARLY = abi.ABSP_STEP_EARLY_PREFETCH
    for x in layers:                                   # warm the flagged variant
        abi.absp_decode_step_ex(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, EARLY, sc)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for x in layers:
            abi.absp_decode_step_ex(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, EARLY, sc)
    stream.synchronize()
    g_plain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_plain, stream=stream):
        for x in layers:
            abi.absp_decode_step(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, sc)
    stream.synchronize()

    def timed(graph, steps, warm):
        for _ in range(warm):
            graph.replay()
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        return reduce_max(e0.elapsed_time(e1), dist, dev)

    with torch.cuda.stream(stream):
        ms, clocks = timed_with_clocks(lambda: timed(g, args.steps, args.warmup),
                                       lambda: ClockSampler(local), dist, dev)
        ms_plain = timed(g_plain, args.steps, args.warmup)
    for x in layers:
        x.check()
    del g_plain
    # the headline layer 0 against the oracle, after its timed launches
    parity = None
    if not args.no_parity and rank == 0:
        parity = parity_record(layers[0], WORKLOAD)

    # incremental tail-row update (one launch per layer); with unchanged
    # lengths it rewrites every tail row with the same bytes
    append = None
    if not args.no_variants:
        ga = torch.cuda.CUDAGraph()
        for x in layers:
            abi.absp_append_centroids(x.kv, x.cent, None, x.ws, sc)
        stream.synchronize()
        with torch.cuda.graph(ga, stream=stream):
            for x in layers:
                abi.absp_append_centroids(x.kv, x.cent, None, x.ws, sc)
        with torch.cuda.stream(stream):
            ms_a = timed(ga, args.steps, args.warmup)
        for x in layers:
            x.check()
        append = {"us_per_layer": ms_a / (args.steps * L) * 1e3,
                  "note": "absp_append_centroids, all 8 KV heads of one layer per launch"}
        del ga
        # the decode loop's own order: each layer's centroid tail update,
        # then its decode step, which may then read nothing before the
        # update completes (the plain step, no early prefetch)
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd, stream=stream):
            for x in layers:
                abi.absp_append_centroids(x.kv, x.cent, None, x.ws, sc)
                abi.absp_decode_step(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, sc)
        with torch.cuda.stream(stream):
            ms_ad = timed(gd, args.steps, args.warmup)
        for x in layers:
            x.check()
        append["then_decode"] = {
            "value": aggregate_rate(world, L, args.steps, ms_ad),
            "us_per_layer": ms_ad / (args.steps * L) * 1e3,
            "note": "per layer: absp_append_centroids then absp_decode_step (plain), the "
                    "sequence a decode loop runs; layer-steps/s"}
        del gd

    # fixed block size for every KV head (the uniform-block methods the page
    # compares against) and unquantised bf16 centroids (its precision
    # baseline), on the same caches, queries and token budget
    fixed = {}
    if not args.no_variants:
        big = abi.LayerKV(  # the largest centroid table: block size 16 everywhere
                          layers[0].data.seq_lens, layers[0].data.page_table,
                          layers[0].data.k_pages, layers[0].data.v_pages,
                          [16] * layers[0].data.num_kv_heads, layers[0].data.num_q_heads)
        fws = abi.alloc_workspace(abi.absp_build_workspace_size(big), dev)
        cases = [(f"fixed_block_{b}", b, abi.ABSP_CENTROIDS_INT4, 0) for b in (16, 32, 64)]
        cases.append(("bf16_centroids", None, abi.ABSP_CENTROIDS_BF16, 0))
        cases.append(("group_max", None, abi.ABSP_CENTROIDS_INT4, abi.ABSP_STEP_GROUP_MAX))
        for name, bsz, fmt, vflags in cases:
            vl = [pipeline.DeviceLayer(
                x.data, stream=sc, fmt=fmt,
                block_size=None if bsz is None else [bsz] * x.data.num_kv_heads)
                for x in layers]
            vb = []
            for y in vl:
                abi.absp_build_centroids(y.kv, fws, sc)
                abi.absp_quantize_centroids(y.kv, fws, y.cent, sc)
                y.score_select(flags=vflags)
                stream.synchronize()
                vb.append(step_bytes(y.data, y.sel.cpu().numpy(), y.sel_count.cpu().numpy(),
                                     y.block_size, fmt == abi.ABSP_CENTROIDS_BF16))
                abi.absp_decode_step_ex(y.kv, y.cent, y.data.q, y.budget, y.out, y.ws,
                                        EARLY | vflags, sc)
            stream.synchronize()
            gv = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gv, stream=stream):
                for y in vl:
                    abi.absp_decode_step_ex(y.kv, y.cent, y.data.q, y.budget, y.out, y.ws,
                                            EARLY | vflags, sc)
            with torch.cuda.stream(stream):
                ms_v = timed(gv, args.steps, args.warmup)
            for y in vl:
                y.check()
            bpl = float(np.mean(vb))
            fixed[name] = {
                "value": aggregate_rate(world, L, args.steps, ms_v),
                "ms_per_step": ms_v / args.steps,
                "bytes_per_launch": bpl,
                "achieved_gbs": bpl / (ms_v / (args.steps * L) * 1e-3) / 1e9}
            del gv, vl
        del fws

    extra = None
    if not args.no_workloads:
        extra = other_workloads(dev, stream, abi, pipeline, synth, timed,
                                args.steps, args.warmup, hbm_peak()[0],
                                parity=not args.no_parity)
        if rank == 0 and not args.no_cpu_baseline:
            for name, cb in oracle_workloads(min(3.0, args.cpu_seconds)).items():
                extra[name]["cpu_baseline"] = cb

    e2e = None
    if not args.no_e2e:
        q_host = [x.data.q.cpu().pin_memory() for x in layers]
        o_host = [torch.empty_like(q).pin_memory() for q in q_host]
        g2 = torch.cuda.CUDAGraph()
        early = abi.ABSP_STEP_EARLY_PREFETCH                # as in the device graph
        for x, qh, oh in zip(layers, q_host, o_host):   # warm outside capture
            abi.absp_decode_step_host_ex(x.kv, x.cent, qh, x.budget, oh, x.ws, early, sc)
        stream.synchronize()
        with torch.cuda.graph(g2, stream=stream):
            for x, qh, oh in zip(layers, q_host, o_host):
                abi.absp_decode_step_host_ex(x.kv, x.cent, qh, x.budget, oh, x.ws, early, sc)
        with torch.cuda.stream(stream):
            ms_e2e = timed(g2, args.steps, args.warmup)
        for x, oh in zip(layers, o_host):
            assert torch.equal(oh.view(torch.int16), x.out.cpu().view(torch.int16))
        qb = sum(q.numel() * 2 for q in q_host)
        e2e = {"value": aggregate_rate(world, L, args.steps, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": qb, "d2h_bytes_per_step": qb,
               "ms_per_step": ms_e2e / args.steps}
        del g2

    # last of the device measurements: independent layer-steps overlapped
    pipelined = None
    if not args.no_variants:
        try:
            ms_p = pipelined_variant(layers, stream, abi, timed, args.steps, args.warmup)
            us_p = ms_p / (args.steps * L) * 1e3
            pipelined = {
                "value": aggregate_rate(world, L, args.steps, ms_p),
                "ms_per_step": ms_p / args.steps, "us_per_launch": us_p,
                "achieved_gbs": bytes_per_launch / (us_p * 1e-6) / 1e9,
                "frac": bytes_per_launch / (us_p * 1e-6) / 1e9 / hbm_peak()[0],
                "streams": PIPELINE_STREAMS,
                "note": "the same layer-steps as independent work on several streams (no "
                        "dependency between them), with ABSP_STEP_THROUGHPUT: a throughput "
                        "mode, not a decode order; the headline keeps the dependent order"}
        except Exception as e:  # the measurements above stand
            pipelined = {"unavailable": f"{type(e).__name__}: {e}"[:200]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        prep, G, budget = oracle_layer_sample(0)
        done, el = time_oracle(prep, G, budget, seconds=args.cpu_seconds)
        cpu = {"value": (done / len(prep)) / el, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{done} (sequence, KV head) decode units of one {WORKLOAD} layer "
                         f"({done / len(prep):.2f} layer-steps, steps 3-5 from prebuilt "
                         f"centroids), numpy fp64, 1 thread, {el:.1f} s"}
        try:
            v, n, units, el2 = time_oracle_all_cores(args.cpu_seconds)
            cpu["all_cores"] = {
                "value": v, "unit": UNIT, "cores": n, "kind": "oracle",
                "sample": f"{units} decode units on {n} processes (one KV head of a "
                          f"{WORKLOAD} layer each, 1 thread each), {el2:.1f} s window"}
        except Exception as e:  # the single-thread figure above stands
            cpu["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
        rb_ms, heads = time_oracle_rebuild(seconds=min(5.0, args.cpu_seconds))
        cpu["rebuild"] = {
            "ms_per_layer": rb_ms, "cores": 1, "kind": "oracle",
            "sample": f"{heads} (sequence, KV head) centroid builds + INT4 quantisations of "
                      f"a {WORKLOAD} layer, numpy fp64, 1 thread (per layer: x Hkv)"}

    peak, peak_kind = hbm_peak()
    launch_ms = ms / (args.steps * L)
    achieved = bytes_per_launch / (launch_ms * 1e-3) / 1e9
    # a launch cannot move its bytes much faster than a plain copy: a figure
    # far above the copy peak means the timed region did not do the work
    if achieved > 1.5 * peak:
        raise RuntimeError(f"implausible launch time {launch_ms * 1e3:.2f} us "
                           f"({achieved:.0f} GB/s for {bytes_per_launch:.0f} B)")
    traffic = recorded_traffic()
    line = {
        "metric": METRIC,
        "value": aggregate_rate(world, L, args.steps, ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(L, world),
        "launch": "CUDA graph of fused score/select/attend launches, PDL, "
                  "ABSP_STEP_EARLY_PREFETCH",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} HBM copy bandwidth",
                     "kernel": "decode_kernel<full>",
                     "bytes_per_launch": bytes_per_launch, "launch_us": launch_ms * 1e3},
        "cpu_baseline": cpu,
        "parity": parity,
        "e2e": e2e,
        "gpu_launches": L * args.steps,
        "variants": {**fixed, "plain": {"value": aggregate_rate(world, L, args.steps, ms_plain),
                               "ms_per_step": ms_plain / args.steps,
                               "note": "absp_decode_step, no reads before the previous "
                                       "launch completes"},
                     **({} if pipelined is None else {"pipelined": pipelined})},
        "append": append,
        "calibration": calib,
        "clocks": clocks,
        "rebuild": {"ms_per_layer": rebuild_ms, "bytes_per_layer": rb_bytes,
                    "achieved_gbs": rb_bytes / (rebuild_ms * 1e-3) / 1e9,
                    "frac": rb_bytes / (rebuild_ms * 1e-3) / 1e9 / peak,
                    "call": "absp_build_quantize_centroids",
                    "two_calls": {"ms_per_layer": rebuild_two_ms,
                                  "frac": rb_bytes / (rebuild_two_ms * 1e-3) / 1e9 / peak,
                                  "call": "absp_build_centroids + absp_quantize_centroids"},
                    "large": None if rb_large is None else
                    {**rb_large, "frac": rb_large["achieved_gbs"] / peak}},
    }
    if extra is not None:
        line["workloads"] = extra
    del g
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
