"""ctypes binding of libabsp (include/absp.h), same names as the C ABI.

Argument marshalling only: torch tensors are turned into raw pointers and
the C structs are filled; every step of the computation runs in the CUDA
library.  Importing this module loads the library and raises if it is
missing -- there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_int32, c_int64, c_size_t,
                    c_uint8, c_uint32, c_void_p)

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("ABSP_LIB", os.path.join(_HERE, "lib", "libabsp.so"))

ABSP_OK = 0
ABSP_ERR_INVALID_ARG = 1
ABSP_ERR_UNSUPPORTED = 2
ABSP_ERR_CUDA = 3
ABSP_ERR_DEVICE_FAULT = 4
ABSP_ERR_TIMEOUT = 5

ABSP_STEP_EARLY_PREFETCH = 1
ABSP_STEP_GROUP_MAX = 2
ABSP_STEP_THROUGHPUT = 4
ABSP_STEP_DIAG_WAIT_TIMEOUT = 0x100
ABSP_CENTROIDS_INT4 = 0
ABSP_CENTROIDS_BF16 = 1

HEAD_DIM = 128
PAGE_SIZE = 16
CODE_ROW_BYTES = 64


class AbspError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        msg = f"{what}: {absp_status_string(status)} (status {status})"
        if self.status == ABSP_ERR_CUDA:   # which CUDA call failed, and how
            self.cuda_error = absp_last_cuda_error()
            msg += f": CUDA error {self.cuda_error} ({absp_last_cuda_error_string()})"
        super().__init__(msg)


class absp_layer_kv(Structure):
    _fields_ = [
        ("num_seqs", c_int32),
        ("num_q_heads", c_int32),
        ("num_kv_heads", c_int32),
        ("head_dim", c_int32),
        ("page_size", c_int32),
        ("max_pages_per_seq", c_int32),
        ("num_phys_pages", c_int64),
        ("seq_lens", c_void_p),
        ("page_table", c_void_p),
        ("k_pages", c_void_p),
        ("v_pages", c_void_p),
        ("block_size", POINTER(c_int32)),
    ]


class absp_centroids(Structure):
    _fields_ = [
        ("codes", POINTER(c_uint8)),
        ("scale", c_void_p),
        ("zp", c_void_p),
        ("format", c_int32),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libabsp.so not found at {LIB_PATH}; build it with "
            "`python -m block_sparse_attention_kv_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    st = c_int32
    P = POINTER
    sig = {
        "absp_status_string": (c_char_p, [st]),
        "absp_build_id": (c_char_p, []),
        "absp_centroid_sizes": (st, [P(absp_layer_kv), P(c_size_t), P(c_size_t), P(c_size_t)]),
        "absp_centroid_sizes_fmt": (st, [P(absp_layer_kv), c_int32, P(c_size_t), P(c_size_t),
                                         P(c_size_t)]),
        "absp_centroid_row_offset": (st, [P(absp_layer_kv), c_int32, c_int32, P(c_int64)]),
        "absp_build_workspace_size": (st, [P(absp_layer_kv), P(c_size_t)]),
        "absp_decode_workspace_size": (st, [P(absp_layer_kv), c_int32, P(c_size_t)]),
        "absp_select_capacity": (st, [P(absp_layer_kv), c_int32, P(c_int32)]),
        "absp_workspace_init": (st, [c_void_p, c_size_t, c_void_p]),
        "absp_build_centroids": (st, [P(absp_layer_kv), c_void_p, c_size_t, c_void_p]),
        "absp_quantize_centroids": (st, [P(absp_layer_kv), c_void_p, c_size_t,
                                         P(absp_centroids), c_void_p]),
        "absp_score_select": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_int32,
                                   c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
        "absp_build_quantize_centroids": (st, [P(absp_layer_kv), c_void_p, c_size_t,
                                               P(absp_centroids), c_void_p]),
        "absp_append_centroids": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_void_p,
                                       c_size_t, c_void_p]),
        "absp_score_select_ex": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_int32,
                                      c_void_p, c_void_p, c_void_p, c_size_t, c_uint32,
                                      c_void_p]),
        "absp_sparse_decode": (st, [P(absp_layer_kv), c_void_p, c_void_p, c_void_p, c_int32,
                                    c_void_p, c_void_p, c_size_t, c_void_p]),
        "absp_decode_step": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_int32,
                                  c_void_p, c_void_p, c_size_t, c_void_p]),
        "absp_decode_step_ex": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_int32,
                                     c_void_p, c_void_p, c_size_t, c_uint32, c_void_p]),
        "absp_decode_step_host": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_int32,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
        "absp_decode_step_host_ex": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p, c_int32,
                                          c_void_p, c_void_p, c_size_t, c_uint32, c_void_p]),
        "absp_check_device_error": (st, [c_void_p, c_size_t, c_void_p, P(c_int32)]),
        "absp_build_quantize_noalloc": (st, [P(absp_layer_kv), P(absp_centroids), c_void_p,
                                             c_void_p]),
        "absp_last_cuda_error": (c_int32, []),
        "absp_last_cuda_error_string": (c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("absp_status_string", "absp_build_id", "absp_centroid_sizes", "absp_centroid_sizes_fmt",
            "absp_centroid_row_offset",
            "absp_build_workspace_size", "absp_decode_workspace_size",
            "absp_select_capacity", "absp_workspace_init", "absp_build_centroids",
            "absp_quantize_centroids", "absp_build_quantize_centroids",
            "absp_append_centroids", "absp_score_select",
            "absp_score_select_ex",
            "absp_sparse_decode",
            "absp_decode_step", "absp_decode_step_ex", "absp_decode_step_host",
            "absp_decode_step_host_ex",
            "absp_check_device_error", "absp_build_quantize_noalloc",
            "absp_last_cuda_error", "absp_last_cuda_error_string")


def lib() -> ctypes.CDLL:
    return _lib


def _check(status: int, what: str) -> None:
    if status != ABSP_OK:
        raise AbspError(status, what)


def _ptr(t) -> int:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _bad(what: str, msg: str):
    raise AbspError(ABSP_ERR_INVALID_ARG, f"{what}: {msg}")


def _arg(t, what: str, name: str, dtype=None, numel: int = 0, where: str = "cuda"):
    """Address of tensor argument `name` of call `what`, after checking what
    the C ABI assumes of the buffer behind it and cannot check itself: its
    element type, a dense row-major layout, its memory space ("cuda": the
    current device; "host": host memory) and at least `numel` elements.
    A raw integer address or None passes through unchecked."""
    if t is None or isinstance(t, int):
        return t
    if not isinstance(t, torch.Tensor):
        _bad(what, f"{name} must be a torch.Tensor or an address")
    if dtype is not None and t.dtype != dtype:
        _bad(what, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        _bad(what, f"{name} must be contiguous")
    if where == "cuda":
        if not t.is_cuda:
            _bad(what, f"{name} must be in device memory")
        if t.device.index != torch.cuda.current_device():
            _bad(what, f"{name} is on cuda:{t.device.index}, the current device is "
                       f"cuda:{torch.cuda.current_device()}")
    elif t.is_cuda:
        _bad(what, f"{name} must be in host memory")
    if t.numel() < numel:
        _bad(what, f"{name} holds {t.numel()} elements, {numel} needed")
    return t.data_ptr()


def _ws(ws, what: str):
    """(address, bytes) of a device workspace tensor."""
    if not isinstance(ws, torch.Tensor):
        _bad(what, "ws must be a device tensor")
    return _arg(ws, what, "ws"), ws.numel() * ws.element_size()


def _qo(kv: "LayerKV") -> int:
    """Elements of a query or output buffer: [S][Hq][128]."""
    return kv.c.num_seqs * kv.c.num_q_heads * HEAD_DIM


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------ structs --

class LayerKV:
    """Owns an absp_layer_kv and keeps the tensors it points at alive."""

    def __init__(self, seq_lens, page_table, k_pages, v_pages, block_size,
                 num_q_heads: int, num_phys_pages: int = None,
                 head_dim: int = HEAD_DIM, page_size: int = PAGE_SIZE):
        self._keep = (seq_lens, page_table, k_pages, v_pages)
        self.block_size = np.ascontiguousarray(np.asarray(block_size, dtype=np.int32))
        self._bs_c = self.block_size.ctypes.data_as(POINTER(c_int32))
        S = int(seq_lens.shape[0]) if seq_lens is not None else 0
        self.c = absp_layer_kv(
            num_seqs=S,
            num_q_heads=int(num_q_heads),
            num_kv_heads=len(self.block_size),
            head_dim=int(head_dim),
            page_size=int(page_size),
            max_pages_per_seq=int(page_table.shape[1]) if page_table is not None else 0,
            num_phys_pages=int(num_phys_pages if num_phys_pages is not None
                               else (k_pages.shape[0] if k_pages is not None else 0)),
            seq_lens=_ptr(seq_lens), page_table=_ptr(page_table),
            k_pages=_ptr(k_pages), v_pages=_ptr(v_pages), block_size=self._bs_c)

    @classmethod
    def from_layer(cls, d) -> "LayerKV":
        """From a synth.LayerData (device tensors)."""
        return cls(d.seq_lens, d.page_table, d.k_pages, d.v_pages, d.block_size,
                   d.num_q_heads)

    @property
    def ref(self):
        return ctypes.byref(self.c)


class Centroids:
    """Owns an absp_centroids over its device tensors."""

    def __init__(self, codes: torch.Tensor, scale: torch.Tensor, zp: torch.Tensor,
                 fmt: int = ABSP_CENTROIDS_INT4):
        self.codes, self.scale, self.zp, self.format = codes, scale, zp, int(fmt)
        self.c = absp_centroids(codes=ctypes.cast(codes.data_ptr(), POINTER(c_uint8)),
                                scale=scale.data_ptr() if scale.numel() else None,
                                zp=zp.data_ptr() if zp.numel() else None, format=int(fmt))

    @property
    def ref(self):
        return ctypes.byref(self.c)


def alloc_centroids(kv: LayerKV, device, fmt: int = ABSP_CENTROIDS_INT4) -> Centroids:
    """Device buffers sized by absp_centroid_sizes_fmt (torch owns the memory)."""
    cb, sb, zb = absp_centroid_sizes_fmt(kv, fmt)
    codes = torch.zeros(max(cb, 256) + 256, dtype=torch.uint8, device=device)
    off = (-codes.data_ptr()) % 256
    codes = codes[off:off + cb]
    scale = torch.zeros(sb // 4, dtype=torch.float32, device=device)
    zp = torch.zeros(zb // 4, dtype=torch.int32, device=device)
    return Centroids(codes, scale, zp, fmt)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled, 256-byte aligned byte buffer."""
    buf = torch.zeros(int(nbytes) + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    return buf[off:off + int(nbytes)]


# ------------------------------------------------------- entry points --

def absp_status_string(status: int) -> str:
    return _lib.absp_status_string(int(status)).decode()


def absp_build_id() -> str:
    """Source hash the loaded library was compiled from."""
    return _lib.absp_build_id().decode()


def absp_last_cuda_error() -> int:
    return int(_lib.absp_last_cuda_error())


def absp_last_cuda_error_string() -> str:
    return _lib.absp_last_cuda_error_string().decode()


def absp_centroid_sizes(kv: LayerKV):
    a, b, c = c_size_t(), c_size_t(), c_size_t()
    _check(_lib.absp_centroid_sizes(kv.ref, ctypes.byref(a), ctypes.byref(b),
                                    ctypes.byref(c)), "absp_centroid_sizes")
    return a.value, b.value, c.value


def absp_centroid_sizes_fmt(kv: LayerKV, fmt: int):
    a, b, c = c_size_t(), c_size_t(), c_size_t()
    _check(_lib.absp_centroid_sizes_fmt(kv.ref, int(fmt), ctypes.byref(a), ctypes.byref(b),
                                        ctypes.byref(c)), "absp_centroid_sizes_fmt")
    return a.value, b.value, c.value


def absp_centroid_row_offset(kv: LayerKV, seq: int, kv_head: int) -> int:
    r = c_int64()
    _check(_lib.absp_centroid_row_offset(kv.ref, int(seq), int(kv_head), ctypes.byref(r)),
           "absp_centroid_row_offset")
    return r.value


def absp_build_workspace_size(kv: LayerKV) -> int:
    r = c_size_t()
    _check(_lib.absp_build_workspace_size(kv.ref, ctypes.byref(r)), "absp_build_workspace_size")
    return r.value


def absp_decode_workspace_size(kv: LayerKV, budget: int) -> int:
    r = c_size_t()
    _check(_lib.absp_decode_workspace_size(kv.ref, int(budget), ctypes.byref(r)),
           "absp_decode_workspace_size")
    return r.value


def absp_select_capacity(kv: LayerKV, budget: int) -> int:
    r = c_int32()
    _check(_lib.absp_select_capacity(kv.ref, int(budget), ctypes.byref(r)),
           "absp_select_capacity")
    return r.value


def absp_workspace_init(ws: torch.Tensor, stream=None) -> None:
    w, wb = _ws(ws, "absp_workspace_init")
    _check(_lib.absp_workspace_init(w, wb, _stream(stream)), "absp_workspace_init")


def _cent(kv: LayerKV, cent: Centroids, what: str):
    """cent.ref after checking its buffers against the layer's sizes."""
    cb, sb, zb = absp_centroid_sizes_fmt(kv, cent.format)
    _arg(cent.codes, what, "codes", torch.uint8, cb)
    if cent.format == ABSP_CENTROIDS_INT4:
        _arg(cent.scale, what, "scale", torch.float32, sb // 4)
        _arg(cent.zp, what, "zp", torch.int32, zb // 4)
    return cent.ref


def _sel(kv: LayerKV, sel, sel_count, budget: int, what: str):
    n = kv.c.num_seqs * kv.c.num_kv_heads
    kmax = absp_select_capacity(kv, budget) if isinstance(sel, torch.Tensor) else 0
    return (_arg(sel, what, "sel", torch.int32, n * kmax),
            _arg(sel_count, what, "sel_count", torch.int32, n))


def absp_build_centroids(kv: LayerKV, ws: torch.Tensor, stream=None) -> None:
    w, wb = _ws(ws, "absp_build_centroids")
    _check(_lib.absp_build_centroids(kv.ref, w, wb, _stream(stream)), "absp_build_centroids")


def absp_quantize_centroids(kv: LayerKV, ws: torch.Tensor, cent: Centroids, stream=None) -> None:
    what = "absp_quantize_centroids"
    w, wb = _ws(ws, what)
    _check(_lib.absp_quantize_centroids(kv.ref, w, wb, _cent(kv, cent, what), _stream(stream)),
           what)


def absp_build_quantize_centroids(kv: LayerKV, ws: torch.Tensor, cent: Centroids,
                                  stream=None) -> None:
    what = "absp_build_quantize_centroids"
    w, wb = _ws(ws, what)
    _check(_lib.absp_build_quantize_centroids(kv.ref, w, wb, _cent(kv, cent, what),
                                              _stream(stream)), what)


def absp_score_select(kv: LayerKV, cent: Centroids, q: torch.Tensor, budget: int,
                      sel: torch.Tensor, sel_count: torch.Tensor, ws: torch.Tensor,
                      stream=None) -> None:
    what = "absp_score_select"
    w, wb = _ws(ws, what)
    sp, cp = _sel(kv, sel, sel_count, budget, what)
    _check(_lib.absp_score_select(kv.ref, _cent(kv, cent, what),
                                  _arg(q, what, "q", torch.bfloat16, _qo(kv)), int(budget),
                                  sp, cp, w, wb, _stream(stream)), what)


def absp_append_centroids(kv: LayerKV, cent: Centroids, exceeded, ws: torch.Tensor,
                          stream=None) -> None:
    what = "absp_append_centroids"
    w, wb = _ws(ws, what)
    ex = _arg(exceeded, what, "exceeded", torch.int32, kv.c.num_seqs * kv.c.num_kv_heads)
    _check(_lib.absp_append_centroids(kv.ref, _cent(kv, cent, what), ex, w, wb,
                                      _stream(stream)), what)


def absp_score_select_ex(kv: LayerKV, cent: Centroids, q: torch.Tensor, budget: int,
                         sel: torch.Tensor, sel_count: torch.Tensor, ws: torch.Tensor,
                         flags: int, stream=None) -> None:
    what = "absp_score_select_ex"
    w, wb = _ws(ws, what)
    sp, cp = _sel(kv, sel, sel_count, budget, what)
    _check(_lib.absp_score_select_ex(kv.ref, _cent(kv, cent, what),
                                     _arg(q, what, "q", torch.bfloat16, _qo(kv)), int(budget),
                                     sp, cp, w, wb, int(flags), _stream(stream)), what)


def absp_sparse_decode(kv: LayerKV, q: torch.Tensor, sel: torch.Tensor,
                       sel_count: torch.Tensor, budget: int, out: torch.Tensor,
                       ws: torch.Tensor, stream=None) -> None:
    what = "absp_sparse_decode"
    w, wb = _ws(ws, what)
    sp, cp = _sel(kv, sel, sel_count, budget, what)
    _check(_lib.absp_sparse_decode(kv.ref, _arg(q, what, "q", torch.bfloat16, _qo(kv)), sp, cp,
                                   int(budget), _arg(out, what, "out", torch.bfloat16, _qo(kv)),
                                   w, wb, _stream(stream)), what)


def absp_decode_step(kv: LayerKV, cent: Centroids, q: torch.Tensor, budget: int,
                     out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    what = "absp_decode_step"
    w, wb = _ws(ws, what)
    _check(_lib.absp_decode_step(kv.ref, _cent(kv, cent, what),
                                 _arg(q, what, "q", torch.bfloat16, _qo(kv)), int(budget),
                                 _arg(out, what, "out", torch.bfloat16, _qo(kv)), w, wb,
                                 _stream(stream)), what)


def absp_decode_step_ex(kv: LayerKV, cent: Centroids, q: torch.Tensor, budget: int,
                        out: torch.Tensor, ws: torch.Tensor, flags: int, stream=None) -> None:
    what = "absp_decode_step_ex"
    w, wb = _ws(ws, what)
    _check(_lib.absp_decode_step_ex(kv.ref, _cent(kv, cent, what),
                                    _arg(q, what, "q", torch.bfloat16, _qo(kv)), int(budget),
                                    _arg(out, what, "out", torch.bfloat16, _qo(kv)), w, wb,
                                    int(flags), _stream(stream)), what)


def absp_decode_step_host(kv: LayerKV, cent: Centroids, q_host: torch.Tensor, budget: int,
                          out_host: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    what = "absp_decode_step_host"
    w, wb = _ws(ws, what)
    _check(_lib.absp_decode_step_host(
        kv.ref, _cent(kv, cent, what),
        _arg(q_host, what, "q_host", torch.bfloat16, _qo(kv), where="host"), int(budget),
        _arg(out_host, what, "out_host", torch.bfloat16, _qo(kv), where="host"), w, wb,
        _stream(stream)), what)


def absp_decode_step_host_ex(kv: LayerKV, cent: Centroids, q_host: torch.Tensor, budget: int,
                             out_host: torch.Tensor, ws: torch.Tensor, flags: int,
                             stream=None) -> None:
    what = "absp_decode_step_host_ex"
    w, wb = _ws(ws, what)
    _check(_lib.absp_decode_step_host_ex(
        kv.ref, _cent(kv, cent, what),
        _arg(q_host, what, "q_host", torch.bfloat16, _qo(kv), where="host"), int(budget),
        _arg(out_host, what, "out_host", torch.bfloat16, _qo(kv), where="host"), w, wb,
        int(flags), _stream(stream)), what)


def absp_build_quantize_noalloc(kv: LayerKV, cent: Centroids, device_status=None,
                                stream=None) -> None:
    """Centroid build + INT4 quantisation without a caller workspace (the
    library's static scratch array is used instead)."""
    what = "absp_build_quantize_noalloc"
    _check(_lib.absp_build_quantize_noalloc(
        kv.ref, _cent(kv, cent, what),
        _arg(device_status, what, "device_status", torch.int32, 2), _stream(stream)), what)


def absp_check_device_error(ws: torch.Tensor, stream=None):
    """Returns (status, detail); status is ABSP_OK when no device fault."""
    d = c_int32()
    w, wb = _ws(ws, "absp_check_device_error")
    st = _lib.absp_check_device_error(w, wb, _stream(stream), ctypes.byref(d))
    if st == ABSP_ERR_CUDA or st == ABSP_ERR_INVALID_ARG:
        raise AbspError(st, "absp_check_device_error")
    return st, d.value
