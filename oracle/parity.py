"""Comparison of CUDA-library results with the CPU oracle.

TEST INFRASTRUCTURE ONLY (used by the tests, the smoke check and the
benchmark's CPU-baseline leg).  The bars:

* INT4 codes, zero points and (bitwise) fp32 scales: exact;
* selected block indices: exact, except pairs that straddle the K boundary
  whose oracle scores lie within 1e-4 * |boundary score| of the boundary
  (GPU scores are fp32, the oracle's fp64); such pairs are counted;
* attention outputs (bf16 out, fp32 accumulation): max |diff| <= 2e-2 and
  mean |diff| <= 2e-3 against the oracle run on the GPU's own selection.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import absp_oracle as O

TIE_REL = 1e-4
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3


@dataclass
class Report:
    heads: int = 0
    code_mismatch: int = 0
    param_mismatch: int = 0
    sel_mismatch: int = 0          # mismatches that are not near-ties
    near_ties: int = 0             # counted boundary near-ties
    out_max_abs: float = 0.0
    out_mean_abs: float = 0.0
    notes: list = field(default_factory=list)

    def ok(self) -> bool:
        return (self.code_mismatch == 0 and self.param_mismatch == 0 and
                self.sel_mismatch == 0 and self.out_max_abs <= OUT_MAX_ABS and
                self.out_mean_abs <= OUT_MEAN_ABS)

    def summary(self) -> str:
        return (f"heads={self.heads} code_mismatch={self.code_mismatch} "
                f"param_mismatch={self.param_mismatch} sel_mismatch={self.sel_mismatch} "
                f"near_ties={self.near_ties} out_max_abs={self.out_max_abs:.3e} "
                f"out_mean_abs={self.out_mean_abs:.3e}")


def compare_codes(rep: Report, hr: O.HeadResult, packed_gpu: np.ndarray,
                  scale_gpu: np.ndarray, zp_gpu: np.ndarray) -> None:
    n = hr.centroids.shape[0]
    want = O.pack_codes(hr.quant.codes)
    got = np.asarray(packed_gpu, dtype=np.uint8).reshape(n, 64)
    bad = int(np.count_nonzero(got != want))
    rep.code_mismatch += bad
    sw = hr.quant.scale.view(np.uint32)
    sg = np.asarray(scale_gpu, dtype=np.float32).view(np.uint32)
    rep.param_mismatch += int(np.count_nonzero(sw != sg))
    rep.param_mismatch += int(np.count_nonzero(hr.quant.zp != np.asarray(zp_gpu)))
    if bad:
        rep.notes.append(f"codes differ in {bad} bytes")


def compare_bf16_centroids(rep: Report, hr: O.HeadResult, rows_gpu: np.ndarray) -> None:
    """BF16 centroid rows (256 bytes each) against the oracle's rounding."""
    n = hr.centroids.shape[0]
    want = O.bf16_bits_of(O.round_bf16(hr.centroids))
    got = np.ascontiguousarray(np.asarray(rows_gpu, dtype=np.uint8).reshape(n, 256)) \
        .view(np.uint16).reshape(n, 128)
    bad = int(np.count_nonzero(got != want))
    rep.code_mismatch += bad
    if bad:
        rep.notes.append(f"bf16 centroids differ in {bad} channels")


def compare_selection(rep: Report, hr: O.HeadResult, sel_gpu) -> None:
    got = [int(x) for x in sel_gpu]
    want = hr.sel.tolist()
    if len(got) != len(want) or got != sorted(got):
        rep.sel_mismatch += max(1, abs(len(got) - len(want)))
        rep.notes.append(f"selection length/order wrong: {len(got)} vs {len(want)}")
        return
    a, b = set(got), set(want)
    if a == b:
        return
    sc = hr.scores
    boundary = np.sort(sc)[::-1][hr.k - 1]
    tol = TIE_REL * abs(boundary) + 1e-12
    for x in a ^ b:
        if abs(sc[x] - boundary) <= tol:
            rep.near_ties += 1
        else:
            rep.sel_mismatch += 1
            rep.notes.append(f"block {x}: score {sc[x]!r} vs boundary {boundary!r}")


def compare_outputs(rep: Report, out_gpu: np.ndarray, out_ref: np.ndarray) -> None:
    d = np.abs(np.asarray(out_gpu, dtype=np.float64) - out_ref)
    rep.out_max_abs = max(rep.out_max_abs, float(d.max()) if d.size else 0.0)
    rep.out_mean_abs = max(rep.out_mean_abs, float(d.mean()) if d.size else 0.0)
