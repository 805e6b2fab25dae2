"""C-ABI library: loads, exports every declared symbol, validates on the host.

No test here launches device work: each call either is pure host logic or
returns an argument error before any CUDA call.
"""

import ctypes
import os
import re

import pytest
import torch

from block_sparse_attention_kv_b200 import build as absp_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def abi():
    absp_build.build()
    from block_sparse_attention_kv_b200 import abi as m
    return m


def _declared_symbols():
    txt = open(os.path.join(ROOT, "include", "absp.h")).read()
    return sorted(set(re.findall(
        r"^\s*(?:ABSP_API\s+)?(?:absp_status|const char\*|int)\s+(absp_\w+)\(", txt, re.M)))


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for want in ("absp_build_centroids", "absp_quantize_centroids", "absp_score_select",
                 "absp_sparse_decode", "absp_decode_step"):
        assert want in names


def test_last_cuda_error_starts_clear(abi):
    # per thread; a thread that has seen no CUDA failure reads 0 / "no error"
    import threading
    seen = []
    t = threading.Thread(target=lambda: seen.append((abi.absp_last_cuda_error(),
                                                     abi.absp_last_cuda_error_string())))
    t.start()
    t.join()
    assert seen == [(0, "no error")]


def test_library_exports_every_declared_symbol(abi):
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(_declared_symbols()) == set(abi.EXPORTED)


def _kv(abi, **over):
    # fake (never dereferenced) device addresses, 256-byte aligned
    args = dict(seq_lens=0x10000, page_table=0x20000, k_pages=0x100000,
                v_pages=0x200000, block_size=[16, 64], num_q_heads=8,
                num_phys_pages=512)
    args.update(over)
    kv = abi.LayerKV(None, None, None, None, args["block_size"], args["num_q_heads"],
                     num_phys_pages=args["num_phys_pages"])
    kv.c.num_seqs = over.get("num_seqs", 1)
    kv.c.max_pages_per_seq = over.get("max_pages", 512)
    kv.c.seq_lens = args["seq_lens"]
    kv.c.page_table = args["page_table"]
    kv.c.k_pages = args["k_pages"]
    kv.c.v_pages = args["v_pages"]
    kv.c.head_dim = over.get("head_dim", 128)
    kv.c.page_size = over.get("page_size", 16)
    return kv


def test_sizes_follow_the_layout(abi):
    kv = _kv(abi)
    codes, scale, zp = abi.absp_centroid_sizes(kv)
    # 8192 tokens: 512 rows at bs 16 + 128 rows at bs 64, 64 B each
    assert codes == (512 + 128) * 64
    assert scale == zp == 2 * 128 * 4
    assert abi.absp_centroid_row_offset(kv, 0, 1) == 512
    kv3 = _kv(abi, num_seqs=3)
    assert abi.absp_centroid_row_offset(kv3, 2, 1) == 2 * 640 + 512
    assert abi.absp_select_capacity(kv, 1024) == 64
    assert abi.absp_select_capacity(kv, 40) == 2          # max(1, 40/16)
    ws = abi.absp_build_workspace_size(kv)
    assert ws == 256 + 2 * 2 * 128 * 8 + 640 * 128 * 8
    assert abi.absp_centroid_sizes_fmt(kv, abi.ABSP_CENTROIDS_INT4) == (codes, scale, zp)
    assert abi.absp_centroid_sizes_fmt(kv, abi.ABSP_CENTROIDS_BF16) == (640 * 256, 0, 0)
    with pytest.raises(abi.AbspError):
        abi.absp_centroid_sizes_fmt(kv, 7)


@pytest.mark.parametrize("over,status", [
    (dict(head_dim=64), 2),
    (dict(page_size=32), 2),
    (dict(block_size=[16, 48]), 1),
    (dict(num_q_heads=7), 1),
    (dict(num_q_heads=2 * 17), 2),          # group of 17 > 16
    (dict(k_pages=0x100010), 1),            # not 256-byte aligned
    (dict(seq_lens=0), 1),
    (dict(num_phys_pages=1 << 27), 2),      # 2^27 pages x 2 heads x 16 rows = 2^32
    (dict(num_phys_pages=1 << 60), 2),      # would wrap the row count
])
def test_invalid_layers_are_rejected(abi, over, status):
    kv = _kv(abi, **over)
    with pytest.raises(abi.AbspError) as e:
        abi.absp_centroid_sizes(kv)
    assert e.value.status == status


def test_misaligned_pages_rejected_by_decode_calls(abi):
    kv = _kv(abi, k_pages=0x100010)
    # a fake, aligned and large enough workspace address: only the page
    # alignment can fail
    st = abi.lib().absp_build_centroids(kv.ref, 0x400000, 1 << 20, None)
    assert st == abi.ABSP_ERR_INVALID_ARG


def test_budget_limits(abi):
    kv = _kv(abi)
    for b in (0, 8, 15, 70000):
        with pytest.raises(abi.AbspError) as e:
            abi.absp_select_capacity(kv, b)
        assert e.value.status == abi.ABSP_ERR_INVALID_ARG


def test_small_workspace_rejected_before_launch(abi):
    kv = _kv(abi)
    st = abi.lib().absp_build_centroids(kv.ref, 0x400000, 64, None)
    assert st == abi.ABSP_ERR_INVALID_ARG


def test_binding_checks_tensor_arguments(abi):
    # what the C ABI cannot see behind a raw pointer is checked by the
    # binding before the call: element type, dense layout, memory space and
    # element count; raw addresses pass through unchecked
    q = torch.zeros((2, 8, 128), dtype=torch.bfloat16)
    assert abi._arg(q, "f", "q", torch.bfloat16, q.numel(), where="host") == q.data_ptr()
    assert abi._arg(0x1000, "f", "q", torch.bfloat16, 1 << 30) == 0x1000
    assert abi._arg(None, "f", "q", torch.bfloat16, 1) is None
    cases = [
        (dict(t=q.float()), "bfloat16"),
        (dict(t=q.transpose(0, 1)), "contiguous"),
        (dict(t=q, numel=q.numel() + 1), "elements"),
        (dict(t=q, where="cuda"), "device memory"),
        (dict(t=[1, 2]), "torch.Tensor"),
    ]
    for kw, text in cases:
        args = dict(dtype=torch.bfloat16, numel=q.numel(), where="host")
        args.update(kw)
        t = args.pop("t")
        with pytest.raises(abi.AbspError) as e:
            abi._arg(t, "f", "q", **args)
        assert e.value.status == abi.ABSP_ERR_INVALID_ARG
        assert text in str(e.value) and "q" in str(e.value)


def test_public_calls_refuse_host_tensors_for_device_buffers(abi):
    kv = _kv(abi)
    with pytest.raises(abi.AbspError) as e:
        abi.absp_build_centroids(kv, torch.zeros(1 << 20, dtype=torch.uint8))
    assert e.value.status == abi.ABSP_ERR_INVALID_ARG
    assert "ws must be in device memory" in str(e.value)


def test_unknown_step_flags_rejected(abi):
    kv = _kv(abi)
    lib = abi.lib()
    st = lib.absp_decode_step_ex(kv.ref, None, None, 1024, None, None, 0, 0x80, None)
    assert st == abi.ABSP_ERR_INVALID_ARG
    st = lib.absp_score_select_ex(kv.ref, None, None, 1024, None, None, None, 0,
                                  abi.ABSP_STEP_EARLY_PREFETCH, None)
    assert st == abi.ABSP_ERR_INVALID_ARG
    st = lib.absp_decode_step_host_ex(kv.ref, None, None, 1024, None, None, 0, 0x80, None)
    assert st == abi.ABSP_ERR_INVALID_ARG


def test_null_layer_and_status_strings(abi):
    lib = abi.lib()
    assert lib.absp_centroid_sizes(None, None, None, None) == abi.ABSP_ERR_INVALID_ARG
    assert abi.absp_status_string(0) == "ok"
    assert "bounds" in abi.absp_status_string(abi.ABSP_ERR_DEVICE_FAULT)
    assert abi.absp_status_string(99) == "unknown status"


def test_build_id_names_the_current_sources(abi):
    # build() reuses a library only when it was compiled from the current
    # sources, and the library carries that source hash
    assert abi.LIB_PATH == absp_build.LIB or os.environ.get("ABSP_LIB")
    assert abi.absp_build_id() == absp_build.source_hash()
    assert absp_build.built_id() == absp_build.source_hash()
