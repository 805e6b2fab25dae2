"""Device buffers + ABI calls for one layer (no arithmetic of its own).

`DeviceLayer` owns the centroid store and the workspaces of one paged layer
and exposes the five library steps; tests, the smoke check and the
benchmark all drive the library through it.
"""

from __future__ import annotations

import torch

from . import abi


class DeviceLayer:
    def __init__(self, data, budget: int = None, stream=None, block_size=None,
                 fmt: int = abi.ABSP_CENTROIDS_INT4):
        """`data` is a synth.LayerData on a CUDA device; `block_size`
        overrides its per-KV-head block-size table (same cache, other
        blocking)."""
        self.data = data
        self.device = data.q.device
        self.budget = int(budget if budget is not None else data.budget)
        self.block_size = list(data.block_size if block_size is None else block_size)
        self.kv = abi.LayerKV(data.seq_lens, data.page_table, data.k_pages, data.v_pages,
                              self.block_size, data.num_q_heads)
        self.cent = abi.alloc_centroids(self.kv, self.device, fmt)
        self.build_ws = None
        dws = abi.absp_decode_workspace_size(self.kv, self.budget)
        self.ws = abi.alloc_workspace(dws, self.device)
        self.kmax = abi.absp_select_capacity(self.kv, self.budget)
        S, Hkv = data.num_seqs, data.num_kv_heads
        self.sel = torch.full((S, Hkv, self.kmax), -1, dtype=torch.int32, device=self.device)
        self.sel_count = torch.zeros((S, Hkv), dtype=torch.int32, device=self.device)
        self.out = torch.zeros_like(data.q)
        self.stream = stream

    # -- steps 1-2 --------------------------------------------------------
    def build_centroids(self, keep_ws: bool = False, fused: bool = False):
        """Steps 1-2: the separate build and quantize calls, or with `fused`
        the single call; both give the same bits."""
        if self.build_ws is None:
            n = abi.absp_build_workspace_size(self.kv)
            self.build_ws = abi.alloc_workspace(n, self.device)
        if fused:
            abi.absp_build_quantize_centroids(self.kv, self.build_ws, self.cent, self.stream)
        else:
            abi.absp_build_centroids(self.kv, self.build_ws, self.stream)
            abi.absp_quantize_centroids(self.kv, self.build_ws, self.cent, self.stream)
        self.check(self.build_ws)
        if not keep_ws:
            self.build_ws = None

    # -- steps 3-5 --------------------------------------------------------
    def score_select(self, q=None, flags: int = 0):
        q = self.data.q if q is None else q
        if flags:
            abi.absp_score_select_ex(self.kv, self.cent, q, self.budget, self.sel,
                                     self.sel_count, self.ws, flags, self.stream)
        else:
            abi.absp_score_select(self.kv, self.cent, q, self.budget, self.sel,
                                  self.sel_count, self.ws, self.stream)

    def sparse_decode(self, q=None, out=None):
        abi.absp_sparse_decode(self.kv, self.data.q if q is None else q, self.sel,
                               self.sel_count, self.budget, self.out if out is None else out,
                               self.ws, self.stream)

    def decode_step(self, q=None, out=None, flags: int = 0):
        q = self.data.q if q is None else q
        out = self.out if out is None else out
        if flags:
            abi.absp_decode_step_ex(self.kv, self.cent, q, self.budget, out, self.ws, flags,
                                    self.stream)
        else:
            abi.absp_decode_step(self.kv, self.cent, q, self.budget, out, self.ws, self.stream)

    def decode_step_host(self, q_host, out_host, flags: int = 0):
        if flags:
            abi.absp_decode_step_host_ex(self.kv, self.cent, q_host, self.budget, out_host,
                                         self.ws, flags, self.stream)
        else:
            abi.absp_decode_step_host(self.kv, self.cent, q_host, self.budget, out_host,
                                      self.ws, self.stream)

    # -- device-side faults ------------------------------------------------
    def check(self, ws=None):
        st, detail = abi.absp_check_device_error(self.ws if ws is None else ws, self.stream)
        if st != abi.ABSP_OK:
            raise abi.AbspError(st, f"device fault (unit {detail})")

    # -- views of the centroid store ----------------------------------------
    def codes_of(self, s: int, h: int, n: int) -> torch.Tensor:
        """Centroid rows of (sequence s, KV head h): [n][64] packed INT4
        codes, or [n][256] bytes of bf16 centroids."""
        rb = 256 if self.cent.format == abi.ABSP_CENTROIDS_BF16 else 64
        r0 = abi.absp_centroid_row_offset(self.kv, s, h)
        return self.cent.codes[r0 * rb:(r0 + n) * rb].view(n, rb)

    def params_of(self, s: int, h: int):
        Hkv = self.data.num_kv_heads
        i = (s * Hkv + h) * 128
        return self.cent.scale[i:i + 128], self.cent.zp[i:i + 128]
