"""CUDA-graph capture of decode steps whose kernels have never run.

A kernel's first launch in a process does one-time set-up (function
attributes, a cluster-fit query).  When that first launch happens inside a
stream capture (torch's default, global capture mode), the set-up must not
touch the capturing stream or the capture is invalidated.  Each case runs in
a fresh process so that the captured launch really is the first of its
kernel instance; the replayed graph must reproduce the eager split path
(score/select, then sparse decode) bit for bit.
"""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import torch
    from block_sparse_attention_kv_b200 import abi, build, pipeline, synth
    build.build()
    flags = {flags}
    host = {host}
    s = torch.cuda.Stream()
    w = synth.custom("capture", 2, 32, 8, [5000, 1777], [16, 32, 64, 16, 32, 64, 16, 32], 512,
                     seed=7)
    layers, refs = [], []
    for i in range(2):
        d = synth.make_layer(w, 0, "cuda")
        d.q.mul_(1.0 + 0.25 * i)                    # distinct queries per layer
        dl = pipeline.DeviceLayer(d, stream=s.cuda_stream)
        dl.build_centroids()
        dl.score_select(flags=flags & abi.ABSP_STEP_GROUP_MAX)
        dl.sparse_decode()
        dl.check()
        torch.cuda.synchronize()
        refs.append(dl.out.clone())
        dl.out.zero_()
        layers.append(dl)
    if host:
        qh = [dl.data.q.cpu().pin_memory() for dl in layers]
        oh = [torch.zeros_like(q).pin_memory() for q in qh]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i, dl in enumerate(layers):
            if host:
                abi.absp_decode_step_host_ex(dl.kv, dl.cent, qh[i], dl.budget, oh[i],
                                             dl.ws, flags, s.cuda_stream)
            else:
                abi.absp_decode_step_ex(dl.kv, dl.cent, dl.data.q, dl.budget, dl.out,
                                        dl.ws, flags, s.cuda_stream)
    torch.cuda.synchronize()
    for rep in range(3):
        for i, dl in enumerate(layers):
            (oh[i] if host else dl.out).zero_()
        g.replay()
        torch.cuda.synchronize()
        for i, dl in enumerate(layers):
            dl.check()
            got = oh[i] if host else dl.out.cpu()
            assert torch.equal(got.view(torch.int16), refs[i].cpu().view(torch.int16)), \\
                ("replay", rep, "layer", i)
    print("ok")
""")


def _run(flags_expr: str, host: bool):
    code = SCRIPT.format(root=ROOT, flags=flags_expr, host=host)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


@pytest.mark.parametrize("flags_expr", [
    "0",
    "abi.ABSP_STEP_EARLY_PREFETCH",
    "abi.ABSP_STEP_EARLY_PREFETCH | abi.ABSP_STEP_GROUP_MAX",
])
def test_cold_capture_device_step(flags_expr):
    _run(flags_expr, host=False)


def test_cold_capture_host_step():
    _run("abi.ABSP_STEP_EARLY_PREFETCH", host=True)
