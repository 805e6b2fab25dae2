"""Property checks of the oracle on generated inputs (hypothesis, CPU).

* top-K: on integer-valued scores (many exact ties) the selection equals the
  definition -- the K best by (score descending, index ascending), listed
  ascending -- computed by brute force over all subsets, for every n <= 10;
* quantiser: on channels of any magnitude (1e-30 .. 1e30, either sign,
  constant channels included) codes stay in 0..15, constant channels are
  degenerate, and every live channel meets the scale/2 dequantisation bound
  (within fp32 rounding of the stored scale) with its minimum at code 0.
"""

import itertools

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import absp_oracle as O


@settings(max_examples=300, deadline=None)
@given(st.lists(st.integers(-4, 4), min_size=1, max_size=10), st.integers(1, 12))
def test_select_is_the_best_subset_with_index_ties(vals, k):
    sc = np.asarray(vals, dtype=np.float64)
    n = len(vals)
    got = O.select_blocks(sc, min(k, n)).tolist()
    kk = min(k, n)
    # best subset: largest score sum; among equal sums the one whose sorted
    # (score desc, index asc) sequence is smallest, which is what "ties to
    # the lower index" means for a set
    def rank_key(sub):
        order = sorted(sub, key=lambda i: (-sc[i], i))
        return (-sum(sc[i] for i in sub), [(-sc[i], i) for i in order])
    best = min(itertools.combinations(range(n), kk), key=rank_key)
    assert got == sorted(best)


magnitudes = st.sampled_from([1e-30, 1e-8, 1e-3, 1.0, 7.0, 1e3, 1e8, 1e30])


@settings(max_examples=150, deadline=None)
@given(st.integers(1, 40), magnitudes, st.floats(-3, 3), st.integers(0, 2 ** 31 - 1))
def test_quantiser_bounds_at_any_magnitude(n, mag, shift, seed):
    rng = np.random.default_rng(seed)
    cent = (rng.standard_normal((n, 128)) + shift) * mag
    cent[:, 7] = shift * mag                         # a constant channel
    q = O.quantize_centroids(cent)
    assert q.codes.min() >= 0 and q.codes.max() <= 15
    assert q.scale[7] == 0 and q.zp[7] == 0 and np.all(q.codes[:, 7] == 0)
    deq = O.dequantize(q)
    live = q.scale > 0
    s = q.scale.astype(np.float64)
    # fp32 rounding of the stored scale moves each level by at most
    # 15 * ulp(scale) / 2; the bound below allows it
    slack = 15 * 2.0 ** -24 * s
    err = np.abs(deq - cent)[:, live]
    assert np.all(err <= (0.5 * s + slack)[live][None, :] + 1e-300)
    mins = np.argmin(cent, axis=0)
    assert np.all(q.codes[mins[live], np.nonzero(live)[0]] == 0)
