"""The failure path of a bounded device wait, made to run out on purpose.

Every mbarrier wait in the decode kernel gives up after a time limit,
records ABSP_ERR_TIMEOUT in the workspace's error word and lets the kernel
carry on to its normal end, so that a lost arrival cannot hang the GPU.
ABSP_STEP_DIAG_WAIT_TIMEOUT launches a kernel instance whose score-exchange
barrier expects 16 bytes that are never sent and whose waits give up after
1 ms: that wait runs out.  The tests check that the launch returns, that the
host reads ABSP_ERR_TIMEOUT with the score wait's site, and that the next
call on the same workspace is clean and correct.  Nothing here faults or
hangs a GPU: all real transfers complete before the wait runs out.
"""

import time

import pytest
import torch

from block_sparse_attention_kv_b200 import synth

pytestmark = pytest.mark.gpu

SCORE_WAIT_SITE = 4   # detail recorded by the score-exchange wait


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, pipeline
    return abi, pipeline


def _layer(lib, w):
    abi, pipeline = lib
    d = synth.make_layer(w, 0, "cuda")
    dl = pipeline.DeviceLayer(d)
    dl.build_centroids()
    return dl


@pytest.mark.parametrize("wname", ["tiny_8k", "llama31_8b_32k"])
def test_score_wait_runs_out_in_the_fused_step(lib, wname):
    abi, _ = lib
    dl = _layer(lib, synth.WORKLOADS[wname])
    dl.decode_step()
    dl.check()
    want = dl.out.clone()
    dl.out.zero_()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dl.decode_step(flags=abi.ABSP_STEP_DIAG_WAIT_TIMEOUT)
    st, detail = abi.absp_check_device_error(dl.ws, dl.stream)   # synchronises
    el = time.perf_counter() - t0
    assert st == abi.ABSP_ERR_TIMEOUT
    assert detail == SCORE_WAIT_SITE
    assert el < 0.5, f"the timed-out launch took {el:.3f} s"
    # the error word was read and cleared: the next call is clean, and its
    # output is the normal one
    dl.out.zero_()
    dl.decode_step()
    st, _ = abi.absp_check_device_error(dl.ws, dl.stream)
    assert st == abi.ABSP_OK
    assert torch.equal(dl.out.view(torch.int16), want.view(torch.int16))


def test_score_wait_runs_out_in_select_only(lib):
    abi, _ = lib
    dl = _layer(lib, synth.WORKLOADS["tiny_8k"])
    dl.score_select()
    dl.check()
    want = dl.sel.clone(), dl.sel_count.clone()
    dl.sel.fill_(-1)
    dl.score_select(flags=abi.ABSP_STEP_DIAG_WAIT_TIMEOUT)
    st, detail = abi.absp_check_device_error(dl.ws, dl.stream)
    assert (st, detail) == (abi.ABSP_ERR_TIMEOUT, SCORE_WAIT_SITE)
    dl.sel.fill_(-1)
    dl.score_select()
    st, _ = abi.absp_check_device_error(dl.ws, dl.stream)
    assert st == abi.ABSP_OK
    assert torch.equal(dl.sel, want[0]) and torch.equal(dl.sel_count, want[1])


def test_diagnostic_flag_is_refused_where_it_has_no_instance(lib):
    abi, _ = lib
    dl = _layer(lib, synth.WORKLOADS["tiny_8k"])
    for extra in (abi.ABSP_STEP_EARLY_PREFETCH, abi.ABSP_STEP_GROUP_MAX):
        with pytest.raises(abi.AbspError) as e:
            dl.decode_step(flags=abi.ABSP_STEP_DIAG_WAIT_TIMEOUT | extra)
        assert e.value.status == abi.ABSP_ERR_UNSUPPORTED
    dl.check()
