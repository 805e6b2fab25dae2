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
       22: "warp 0 ballot words out", 13: "ballot", 14: "ranked", 5: "top-K done",
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
    print("| phase | median CTA (ns) | slowest CTA (ns) |")
    print("|---|---|---|")
    for j in range(2, 11):
        med, mx = [], []
        for k in slots:
            c = Cc[k, :ncta]
            dd = (c[:, j] - c[:, j - 1]) / ghz
            med.append(np.median(dd))
            mx.append(dd.max())
        print(f"| {NAMES[j - 1]} -> {NAMES[j]} | {np.median(med):.0f} | {np.median(mx):.0f} |")
    print()
    print("| stamp (globaltimer from release) | median CTA (ns) | slowest CTA (ns) |")
    print("|---|---|---|")
    for j in range(0, 11):
        med, mx = [], []
        for k in slots:
            t = T[k, :ncta]
            rel = t[:, 1].min()
            v = t[:, j] - rel
            med.append(np.median(v))
            mx.append(v.max())
        print(f"| {NAMES[j]} | {np.median(med):.0f} | {np.median(mx):.0f} |")
    print()
    print("| top-K sub-phase (clock64 from 'all scores') | median CTA (ns) | slowest CTA (ns) |")
    print("|---|---|---|")
    for j, name in SUB.items():
        med, mx = [], []
        for k in slots:
            c = Cc[k, :ncta]
            ok = c[:, j] != 0
            if not ok.any():
                continue
            dd = (c[ok, j] - c[ok, 4]) / ghz
            med.append(np.median(dd))
            mx.append(dd.max())
        if med:
            print(f"| {name} | {np.median(med):.0f} | {np.median(mx):.0f} |")
    print()
    # the same phases by the KV head's block size (CTA i of a launch works
    # on head (i / C) % Hkv, C CTAs per head)
    pairs = layers[0].data.num_seqs * layers[0].data.num_kv_heads
    per_head = max(1, ncta // pairs)
    hkv = layers[0].data.num_kv_heads
    print("| phase | " + " | ".join(f"bs {b}: median CTA (ns)" for b in (16, 32, 64)) + " |")
    print("|---|---|---|---|")
    for j in range(2, 11):
        cols = []
        for b in (16, 32, 64):
            med = []
            for k in slots:
                bsz = np.asarray(layers[k].data.block_size)
                ctas = [i for i in range(ncta) if int(bsz[(i // per_head) % hkv]) == b]
                if not ctas:
                    continue
                c = Cc[k, ctas]
                med.append(np.median((c[:, j] - c[:, j - 1]) / ghz))
            cols.append(f"{np.median(med):.0f}" if med else "-")
        print(f"| {NAMES[j - 1]} -> {NAMES[j]} | " + " | ".join(cols) + " |")
    print()
    print("| scoring sub-phase (clock64 from 'query+weights') | median CTA (ns) | slowest CTA (ns) |")
    print("|---|---|---|")
    for j, name in SCORE.items():
        med, mx = [], []
        for k in slots:
            c = Cc[k, :ncta]
            ok = c[:, j] != 0
            if not ok.any():
                continue
            dd = (c[ok, j] - c[ok, 2]) / ghz
            med.append(np.median(dd))
            mx.append(dd.max())
        if med:
            print(f"| {name} | {np.median(med):.0f} | {np.median(mx):.0f} |")


if __name__ == "__main__":
    main(sys.argv)
