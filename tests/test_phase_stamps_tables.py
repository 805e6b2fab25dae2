"""Host arithmetic of the phase-timeline tool on hand-made stamps.

The decode kernel's profiling build writes, per launch k, CTA i and slot j,
a globaltimer stamp T[k, i, j] (ns) and a clock64 stamp Cc[k, i, j]
(cycles, 0 where the slot was not stamped).  The stamps below are chosen
so that every median and maximum in the tables is known by hand.
"""

import numpy as np

from block_sparse_attention_kv_b200 import phase_stamps as ps

L, NCTA, SLOTS = 8, 16, 24
GHZ = 2.0                      # 2 cycles per ns


def _stamps():
    T = np.zeros((L, NCTA, SLOTS), dtype=np.int64)
    Cc = np.zeros((L, NCTA, SLOTS), dtype=np.int64)
    i = np.arange(NCTA)
    for k in range(L):
        off = 1_000_000 * k                    # cancels in every figure
        T[k, :, 0] = off + 8 * i               # entry: 1050 ns before the release
        for j in range(1, 11):
            T[k, :, j] = off + 1000 + 8 * i + 50 * j
        # CTAs 0..7 (KV head 0) take 100 ns per phase, CTAs 8..15 200 ns
        slow = np.where(i >= 8, 2, 1)
        for j in range(0, 11):
            Cc[k, :, j] = off + 200 * j * slow
        Cc[k, :, 11] = Cc[k, :, 4] + 2 * 30 * (i + 1)      # 30 .. 480 ns after 'all scores'
        Cc[k, :4, 12] = Cc[k, :4, 4] + 2 * 10              # stamped by CTAs 0..3 only
        Cc[k, :, 18] = Cc[k, :, 2] + 2 * 5
    return T, Cc


def _table(lines, title):
    start = next(n for n, l in enumerate(lines) if l.startswith(f"| {title}"))
    rows = {}
    for l in lines[start + 2:]:
        if not l:
            break
        cells = [c.strip() for c in l.strip("|").split("|")]
        rows[cells[0]] = cells[1:]
    return rows


def test_tables_medians_and_maxima():
    T, Cc = _stamps()
    bs = [np.array([16, 64])] * L               # head 0 at bs 16, head 1 at bs 64
    lines = ps.tables(T, Cc, NCTA, GHZ, range(4, L), bs, per_head=8)

    phases = _table(lines, "phase | median CTA")
    assert len(phases) == 9
    # 8 CTAs at 100 ns and 8 at 200 ns: median 150, slowest 200
    assert phases["released -> query+weights"] == ["150", "200"]
    assert phases["cluster merge -> output written"] == ["150", "200"]

    stamps = _table(lines, "stamp (globaltimer")
    # from the earliest release (CTA 0): CTA i is 8 i ns late, median 60, max 120
    assert stamps["released"] == ["60", "120"]
    assert stamps["output written"] == [str(60 + 450), str(120 + 450)]
    assert stamps["entry (before the release: negative)"] == [str(60 - 1050), str(120 - 1050)]

    sub = _table(lines, "top-K sub-phase")
    assert sub["histogram"] == ["255", "480"]   # 30 (i + 1) ns over i = 0..15
    assert sub["boundary bin"] == ["10", "10"]  # only the CTAs that stamped it
    assert "warp 0 histogram issued" not in sub  # never stamped: no row

    by_bs = _table(lines, "phase | bs 16")
    assert by_bs["released -> query+weights"] == ["100", "-", "200"]

    score = _table(lines, "scoring sub-phase")
    assert score["scoring starts"] == ["5", "5"]


def test_median_is_over_the_summarised_launches_only():
    T, Cc = _stamps()
    # a slow launch outside the summarised range changes nothing
    Cc[0, :, 3:] += 2 * 10_000                 # 'own rows scored' 10 us late
    T[0, :, 5:] += 10_000
    bs = [np.array([16, 64])] * L
    a = ps.tables(T, Cc, NCTA, GHZ, range(4, L), bs, per_head=8)
    T2, Cc2 = _stamps()
    b = ps.tables(T2, Cc2, NCTA, GHZ, range(4, L), bs, per_head=8)
    assert a == b
    # inside the range, one launch of three cannot move the median
    Cc[5, :, 3:] += 2 * 10_000
    c = ps.tables(T, Cc, NCTA, GHZ, range(4, 7), bs, per_head=8)
    assert _table(c, "phase | median CTA")["query+weights -> own rows scored"] == ["150", "200"]
