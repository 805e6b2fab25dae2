"""The parity checker itself (oracle/parity.py), on the CPU: the oracle's
own results pass, and each planted mistake of the kind the GPU could make --
a flipped code nibble, a scale one ulp off, a zero point off by one, a wrong
block, a selection out of order or of the wrong length, a bf16 centroid one
bit off, outputs past the tolerance -- is caught; only a boundary near-tie is
let through, and counted."""

import copy

import numpy as np

from block_sparse_attention_kv_b200 import synth
from oracle import absp_oracle as O
from oracle import parity as PR


def _head():
    w = synth.custom("chk", 1, 4, 1, [1500], [16], 256, seed=21)
    hl = synth.host_layer(synth.make_layer(w, 0, "cpu"))
    res = O.run_layer(hl)
    return res, res.heads[(0, 0)]


def _codes_report(hr, packed, scale, zp):
    rep = PR.Report(heads=1)
    PR.compare_codes(rep, hr, packed, scale, zp)
    return rep


def test_codes_and_parameters():
    _, hr = _head()
    packed = O.pack_codes(hr.quant.codes)
    scale, zp = hr.quant.scale.copy(), hr.quant.zp.copy()
    assert _codes_report(hr, packed, scale, zp).ok()
    bad = packed.copy()
    bad[3, 7] ^= 0x10                                # one nibble of one row
    r = _codes_report(hr, bad, scale, zp)
    assert r.code_mismatch == 1 and not r.ok()
    s2 = scale.copy()
    s2[5] = np.nextafter(s2[5], np.float32(np.inf))  # one ulp
    r = _codes_report(hr, packed, s2, zp)
    assert r.param_mismatch == 1 and not r.ok()
    z2 = zp.copy()
    z2[9] += 1
    r = _codes_report(hr, packed, scale, z2)
    assert r.param_mismatch == 1 and not r.ok()


def test_selection():
    _, hr = _head()
    sel = hr.sel.tolist()

    def check(got):
        rep = PR.Report(heads=1)
        PR.compare_selection(rep, hr, got)
        return rep

    assert check(sel).ok()
    # swap the best selected block for the worst unselected one
    out = sorted(set(range(len(hr.scores))) - set(sel), key=lambda b: hr.scores[b])[0]
    best = max(sel, key=lambda b: hr.scores[b])
    r = check(sorted(set(sel) - {best} | {out}))
    assert r.sel_mismatch == 2 and r.near_ties == 0 and not r.ok()
    r = check(sel[::-1])                             # not ascending
    assert r.sel_mismatch >= 1 and not r.ok()
    r = check(sel[:-1])                              # one block short
    assert r.sel_mismatch >= 1 and not r.ok()


def test_boundary_near_tie_is_counted_not_failed():
    _, hr = _head()
    h2 = copy.deepcopy(hr)
    order = np.argsort(-h2.scores, kind="stable")
    last_in, first_out = int(order[h2.k - 1]), int(order[h2.k])
    # move the first unselected score to within 1e-6 (relative) of the boundary
    h2.scores[first_out] = h2.scores[last_in] * (1 - 1e-6 * np.sign(h2.scores[last_in]))
    got = sorted(set(h2.sel.tolist()) - {last_in} | {first_out})
    rep = PR.Report(heads=1)
    PR.compare_selection(rep, h2, got)
    assert rep.near_ties == 2 and rep.sel_mismatch == 0 and rep.ok()


def test_bf16_centroid_rows():
    _, hr = _head()
    want = O.bf16_bits_of(O.round_bf16(hr.centroids))
    rows = want.view(np.uint8).reshape(hr.centroids.shape[0], 256)
    rep = PR.Report(heads=1)
    PR.compare_bf16_centroids(rep, hr, rows)
    assert rep.ok()
    bad = want.copy()
    bad[2, 40] ^= 1
    rep = PR.Report(heads=1)
    PR.compare_bf16_centroids(rep, hr, bad.view(np.uint8).reshape(-1, 256))
    assert rep.code_mismatch == 1 and not rep.ok()


def test_output_tolerances():
    res, _ = _head()
    ref = res.out
    for delta, ok in ((0.0, True), (1.9e-2, True), (2.1e-2, False)):
        got = ref.copy()
        got[0, 1, 3] += delta                        # one element off by delta
        rep = PR.Report(heads=1)
        PR.compare_outputs(rep, got, ref)
        assert rep.ok() is ok, delta
    rep = PR.Report(heads=1)
    PR.compare_outputs(rep, ref + 2.5e-3, ref)       # every element: mean too large
    assert rep.out_max_abs <= PR.OUT_MAX_ABS and not rep.ok()
