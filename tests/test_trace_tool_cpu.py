"""The tracing tool's record decoding and summaries, on synthetic records (no GPU).

A record is two 64-bit words per event: %globaltimer (ns) and (SM clock << 32 | event << 24 |
tile << 16 | k-block), stored per launch slot at [(cta * 4 + role) * ROLE_CAP + i]."""
import numpy as np

from activation_epilogue_tcgen05_b200 import trace as tr


def _slot(records):
    """records: (cta, role, i, globaltimer, clk, ev, tile, kb) -> the two word arrays of one slot."""
    t = np.zeros(tr.LAUNCH_RECS, dtype=np.uint64)
    w = np.zeros(tr.LAUNCH_RECS, dtype=np.uint64)
    for cta, role, i, gt, clk, ev, tile, kb in records:
        j = (cta * 4 + role) * tr.ROLE_CAP + i
        t[j] = gt
        w[j] = (clk << 32) | (ev << 24) | (tile << 16) | kb
    return t, w


def test_records_decode_per_launch_slot():
    t0, w0 = _slot([(3, 1, 0, 1000, 77, 22, 5, 9), (3, 0, 2, 900, 70, 20, 5, 9)])
    t1, w1 = _slot([(0, 2, 0, 5000, 12, 27, 1, 2)])
    L = tr._launches(np.concatenate([t0, t1]), np.concatenate([w0, w1]))
    assert len(L) == 2
    a = L[0]
    order = np.argsort(a["gt"])
    assert a["cta"][order].tolist() == [3, 3] and a["role"][order].tolist() == [0, 1]
    assert a["ev"][order].tolist() == [20, 22] and a["tile"][order].tolist() == [5, 5]
    assert a["kb"][order].tolist() == [9, 9] and a["clk"][order].tolist() == [70, 77]
    assert L[1]["ev"].tolist() == [27] and L[1]["cta"].tolist() == [0] and L[1]["role"].tolist() == [2]


def test_persistent_summary_latency_and_period():
    # one CTA: loads issued at clocks 0, 100, 200; the MMA passes their barriers at 1000, 2000, 3000
    recs = []
    for s in range(3):
        recs.append((0, 0, s, 10 + s, 100 * s, 20, 1, s))
        recs.append((0, 1, s, 1000 + 1000 * s, 1000 + 1000 * s, 22, 1, s))
    recs.append((0, 2, 0, 5000, 5000, 27, 1, 0))
    t, w = _slot(recs)
    lines = tr.summarise_persistent(tr._launches(t, w))
    text = "\n".join(lines)
    # latencies 1000, 1900, 2800; periods 1000, 1000
    assert "p10/p50/p90: 1180 / 1900 / 2620" in text
    assert "MMA issuer period between stages (SM clocks) p10/p50/p90: 1000 / 1000 / 1000; mean 1000" in text


def test_cluster_phases_split_by_rank():
    # two CTAs of one cluster (rank 0 and 1): release at 0, last MMA at 5 us, accumulator at
    # 5.1, partials in at 5.6 (rank 0) / 5.7, epilogue done 6.0 / 6.1, end 6.3 / 6.4
    recs = []
    for cta, rank, extra in ((0, 0, 0), (1, 1, 100)):
        recs += [(cta, 0, 0, 1, 1, 11, 0, rank),          # (a zero timer word marks an empty record)
                 (cta, 1, 0, 5000, 9000, 23, 0, 16),
                 (cta, 2, 0, 5100, 9200, 26, 0, rank),
                 (cta, 2, 1, 5600 + extra, 10200 + extra, 28, 0, rank),
                 (cta, 2, 2, 6000 + extra, 11000 + extra, 27, 0, rank),
                 (cta, 3, 0, 6300 + extra, 11600 + extra, 29, 0, rank)]
    t, w = _slot(recs)
    (L,) = tr._launches(t, w)
    text = "\n".join(tr._cluster_phases(L))
    assert "cluster size 2" in text
    assert "accumulator ready -> partials received" in text
    line = next(s for s in text.splitlines() if "partials received -> epilogue done" in s and "rank 0" in s)
    assert "0.40" in line and "clocks 800" in line
