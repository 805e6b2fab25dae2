"""Per-head block-size sensitivity calibration and block-size allocation.

CPU: the oracle's recall count and its invariants, and the library's exact
allocation against an exhaustive search.  GPU: the library's calibration
(its own kernels select at every block size) against the oracle's, count
for count, and the allocation drawn from it.
"""

import numpy as np
import pytest

from block_sparse_attention_kv_b200 import synth
from oracle import calibration as OC


def _small(budget=512, seed=90):
    # 4 KV heads whose 128 relevant tokens come in spans of 4, 16, 64, 256
    return synth.custom("calib_small", 1, 16, 4, [8192], [16] * 4, budget, seed=seed,
                        planted_lens=(4, 16, 64, 256), planted_tokens=128)


def _relevant(d):
    return lambda s, h: synth.planted_mask(d.plan, s, h)


# ------------------------------------------------------------- oracle pins --

def test_token_hits_by_hand():
    rel = np.zeros(100, bool)
    rel[[0, 15, 16, 40, 99]] = True
    assert OC.token_hits([0], 16, 100, rel) == 2          # tokens 0, 15
    assert OC.token_hits([1, 6], 16, 100, rel) == 2       # 16; 99 in the short block 6
    assert OC.token_hits([2], 32, 100, rel) == 0          # tokens 64..95
    assert OC.token_hits([1], 32, 100, rel) == 1          # 40
    assert OC.token_hits([], 16, 100, rel) == 0


def test_normalised_recall_definition():
    hits = np.array([[8, 4, 2], [0, 0, 0], [5, 5, 6]])
    rel = np.array([10, 10, 0])
    nr = OC.normalised_recall(hits, rel)
    assert np.allclose(nr[0], [1.0, 0.5, 0.25])
    assert np.all(nr[1] == 1.0) and np.all(nr[2] == 1.0)  # no recall at 16 / nothing relevant


def test_budget_covering_the_context_recalls_everything():
    # K = all blocks at every block size: every relevant token is selected
    d = synth.make_layer(_small(budget=8192), 0, "cpu")
    hits, rel, rows = OC.calibrate(synth.host_layer(d), _relevant(d))
    assert np.array_equal(hits, np.repeat(rel[:, None], 3, axis=1))
    assert np.array_equal(rows[0], [512, 256, 128])


def test_concentrated_heads_lose_recall_as_blocks_grow():
    # the premise of the sensitivity analysis, on this seeded set: a head
    # whose relevant keys come in 4-token spans keeps little of its recall
    # at block size 64, one with 256-token spans keeps all of it
    d = synth.make_layer(_small(), 0, "cpu")
    hits, rel, _ = OC.calibrate(synth.host_layer(d), _relevant(d))
    nr = OC.normalised_recall(hits, rel)
    assert np.all(nr[:, 0] == 1.0)
    assert nr[0, 2] < 0.5
    assert nr[3, 2] >= 0.95


# ------------------------------------------------------- host allocation --

def test_allocation_matches_exhaustive_search():
    from block_sparse_attention_kv_b200.calibrate import allocate
    rng = np.random.default_rng(7)
    for _ in range(400):
        H = int(rng.integers(1, 6))
        value = np.round(rng.random((H, 3)), int(rng.integers(1, 3)))  # ties happen
        cost = rng.integers(1, 20, size=(H, 3))
        budget = int(rng.integers(0, 60))
        assert allocate(value, cost, budget) == OC.best_allocation(value, cost, budget)


def test_allocation_without_room_is_reported():
    from block_sparse_attention_kv_b200.calibrate import allocate
    choice, v, c = allocate(np.ones((2, 3)), np.full((2, 3), 10), 15)
    assert choice is None and v == -np.inf


def test_selected_token_mask_by_hand():
    from block_sparse_attention_kv_b200.calibrate import selected_token_mask
    m = selected_token_mask(np.array([1, 6, 3]), 2, 16, 100)  # the third entry is not counted
    want = np.zeros(100, bool)
    want[16:32] = True
    want[96:100] = True
    assert np.array_equal(m, want)


# --------------------------------------------------------------- GPU parity --

@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_kv_b200 import build
    build.build()
    from block_sparse_attention_kv_b200 import abi, calibrate
    return abi, calibrate


@pytest.mark.gpu
def test_calibration_matches_oracle(lib):
    _, cal = lib
    w = _small()
    d = synth.make_layer(w, 0, "cuda")
    got = cal.calibrate(d, _relevant(d))
    hits, rel, rows = OC.calibrate(synth.host_layer(d), _relevant(d))
    assert np.array_equal(got.hits, hits), (got.hits, hits)
    assert np.array_equal(got.relevant, rel)
    assert np.array_equal(got.rows, rows)
    nr = OC.normalised_recall(hits, rel)
    assert np.array_equal(got.normalised, nr)
    budget = int(rows[:, 1].sum())           # the centroid store of uniform bs 32
    assert cal.allocate(got.normalised, got.rows, budget) == \
        OC.best_allocation(nr, rows, budget)


@pytest.mark.gpu
def test_calibration_llama_shaped_heads(lib):
    # the benchmark's calibration set: 8 heads, spans of 4 .. 512 tokens, 32K
    _, cal = lib
    w = synth.WORKLOADS["calib_8h_32k"]
    d = synth.make_layer(w, 0, "cuda")
    got = cal.calibrate(d, _relevant(d))
    hits, rel, rows = OC.calibrate(synth.host_layer(d), _relevant(d))
    assert np.array_equal(got.hits, hits), (got.hits, hits)
    nr = got.normalised
    assert nr[0, 2] < nr[7, 2]                # 4-token spans lose more than 512
