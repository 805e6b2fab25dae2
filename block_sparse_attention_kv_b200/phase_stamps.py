"""Phase timeline of the fused decode kernel, from the profiling build.

    python -m block_sparse_attention_kv_b200.phase_stamps [workload] [layers]

Builds the separate library with the decode kernel's phase stamps
(ABSP_PHASE_STAMPS; the product library has none), replays `layers`
distinct layer caches of `workload` as one CUDA graph of dependent
launches (programmatic dependent launch, early prefetch), as the benchmark
does, and prints, per phase, the median over launches of the median and
the slowest CTA: clock64 deltas between consecutive stamps, and
globaltimer times from the moment the preceding launch released the CTAs.
The stamps cost a few hundred nanoseconds per launch; the benchmark's own
figure comes from the product library.
"""

from __future__ import annotations

import ctypes
import json
import os
import sys

import numpy as np

from . import build

NAMES = {0: "entry (before the release: negative)", 1: "released", 2: "query+weights", 3: "own rows scored",
         4: "all scores", 5: "top-K", 6: "1st page landed", 7: "attended",
         8: "warp merge", 9: "cluster merge", 10: "output written"}
SUB = {21: "warp 0 histogram issued", 11: "histogram", 12: "boundary bin",
       22: "warp 0 selection words out", 13: "selection words and candidates", 14: "ranked", 5: "top-K done",
       16: "barrier", 17: "page ids", 23: "proxy fence", 15: "copies issued"}
SCORE = {18: "scoring starts", 19: "first code stage here", 20: "warp 0 scored first stage",
         3: "own rows scored"}


def main(argv) -> None:
    wname = argv[1] if len(argv) > 1 else "llama31_8b_32k"
    L = int(argv[2]) if len(argv) > 2 else 64
    lib_path = build.build(stamps=True)
    os.environ["ABSP_LIB"] = lib_path
    import torch
    from . import abi, pipeline, synth
    if os.path.realpath(abi.LIB_PATH) != os.path.realpath(lib_path):
        raise RuntimeError("the binding was imported before the profiling library was chosen")
    lib = ctypes.CDLL(lib_path)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flags = abi.ABSP_STEP_EARLY_PREFETCH
    w = synth.WORKLOADS[wname]
    stream = torch.cuda.Stream(device=dev)
    sc = stream.cuda_stream
    layers = []
    with torch.cuda.stream(stream):
        for i in range(L):
            x = pipeline.DeviceLayer(synth.make_layer(w, i, dev), stream=sc)
            x.build_centroids()
            layers.append(x)
    stream.synchronize()
    for x in layers:
        abi.absp_decode_step_ex(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, flags, sc)
    stream.synchronize()
    lib.absp_phase_stamps_reset()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for x in layers:
            abi.absp_decode_step_ex(x.kv, x.cent, x.data.q, x.budget, x.out, x.ws, flags, sc)
    with torch.cuda.stream(stream):
        for _ in range(5):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        steps = 50
        e0.record(stream)
        for _ in range(steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / (steps * L) * 1e3
    for x in layers:
        x.check()
    T = np.zeros(64 * 160 * 24, dtype=np.uint64)
    Cc = np.zeros(64 * 160 * 24, dtype=np.int64)
    rc = lib.absp_phase_stamps_copy(T.ctypes.data_as(ctypes.c_void_p),
                                    Cc.ctypes.data_as(ctypes.c_void_p))
    if rc != 0:
        raise RuntimeError(f"stamp copy failed ({rc})")
    T = T.reshape(64, 160, 24).astype(np.int64)
    Cc = Cc.reshape(64, 160, 24)
    ncta = 0
    while ncta < 160 and T[0, ncta, 0] != 0:
        ncta += 1
    ghz = None
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(0)
        ghz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM) / 1e3
    except Exception:
        ghz = 1.965
    slots = range(4, min(L, 64))
    print(json.dumps({"workload": wname, "layers": L, "us_per_launch_stamped": round(us, 3),
                      "ctas": ncta, "sm_ghz": ghz, "build_id": abi.absp_build_id()}))
    pairs = layers[0].data.num_seqs * layers[0].data.num_kv_heads
    block_sizes = [np.asarray(layers[k].data.block_size) for k in range(L)]
    for line in tables(T, Cc, ncta, ghz, slots, block_sizes, max(1, ncta // pairs)):
        print(line)


def _row(name: str, med: list, mx: list) -> str:
    return f"| {name} | {np.median(med):.0f} | {np.median(mx):.0f} |"


def tables(T, Cc, ncta: int, ghz: float, slots, block_sizes, per_head: int) -> list[str]:
    """The timeline tables as markdown lines.

    T[k, i, j] is the globaltimer stamp (ns) and Cc[k, i, j] the clock64
    stamp of slot j by CTA i in launch k (0 where the slot was not
    stamped); `slots` are the launches summarised; block_sizes[k] is launch
    k's per-KV-head block-size table, and CTA i works on KV head
    (i // per_head) % len(block_sizes[k]).  Each figure is the median over
    the launches of the median CTA and of the slowest CTA.
    """
    out = ["| phase | median CTA (ns) | slowest CTA (ns) |", "|---|---|---|"]
    for j in range(2, 11):
        med, mx = [], []
        for k in slots:
            dd = (Cc[k, :ncta, j] - Cc[k, :ncta, j - 1]) / ghz
            med.append(np.median(dd))
            mx.append(dd.max())
        out.append(_row(f"{NAMES[j - 1]} -> {NAMES[j]}", med, mx))
    out += ["", "| stamp (globaltimer from release) | median CTA (ns) | slowest CTA (ns) |",
            "|---|---|---|"]
    for j in range(0, 11):
        med, mx = [], []
        for k in slots:
            t = T[k, :ncta]
            v = t[:, j] - t[:, 1].min()
            med.append(np.median(v))
            mx.append(v.max())
        out.append(_row(NAMES[j], med, mx))

    def sub_table(title: str, names: dict, origin: int) -> list[str]:
        rows = ["", f"| {title} | median CTA (ns) | slowest CTA (ns) |", "|---|---|---|"]
        for j, name in names.items():
            med, mx = [], []
            for k in slots:
                c = Cc[k, :ncta]
                ok = c[:, j] != 0
                if not ok.any():
                    continue
                dd = (c[ok, j] - c[ok, origin]) / ghz
                med.append(np.median(dd))
                mx.append(dd.max())
            if med:
                rows.append(_row(name, med, mx))
        return rows

    out += sub_table("top-K sub-phase (clock64 from 'all scores')", SUB, 4)
    sizes = (16, 32, 64)
    out += ["", "| phase | " + " | ".join(f"bs {b}: median CTA (ns)" for b in sizes) + " |",
            "|---|---|---|---|"]
    for j in range(2, 11):
        cols = []
        for b in sizes:
            med = []
            for k in slots:
                bsz = block_sizes[k]
                ctas = [i for i in range(ncta) if int(bsz[(i // per_head) % len(bsz)]) == b]
                if ctas:
                    c = Cc[k, ctas]
                    med.append(np.median((c[:, j] - c[:, j - 1]) / ghz))
            cols.append(f"{np.median(med):.0f}" if med else "-")
        out.append(f"| {NAMES[j - 1]} -> {NAMES[j]} | " + " | ".join(cols) + " |")
    out += sub_table("scoring sub-phase (clock64 from 'query+weights')", SCORE, 2)
    return out

if __name__ == "__main__":
    main(sys.argv)
