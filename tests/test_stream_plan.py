"""The ring-stream plan of the oracle, against a brute-force ring simulation and
the grouping rules it states (macrobatches of two waves that fit in the ring)."""
import numpy as np
import pytest

import oracle as O


def _simulate(plan, ring_rows):
    """Write every segment into a ring of owner ids; resident = still fully owned."""
    owner = np.full(ring_rows, -1)
    for m, (s, n) in enumerate(zip(plan["ring_start"], plan["sizes"])):
        assert 0 <= s and s + n <= ring_rows
        owner[s:s + n] = m
    return [bool(np.all(owner[s:s + n] == m)) for m, (s, n) in enumerate(zip(plan["ring_start"], plan["sizes"]))]


@pytest.mark.parametrize("seed,M,El,scale,ring,min_rows", [
    (0, 16, 6, 300, 18724 // 4, 2368), (1, 16, 6, 900, 18724, 2368), (2, 8, 3, 50, 2000, 1024),
    (3, 12, 5, 2000, 18724, 2368), (4, 5, 2, 0, 1000, 512), (5, 16, 6, 3000, 18724, 2368)])
def test_plan_matches_ring_simulation_and_grouping_rules(seed, M, El, scale, ring, min_rows):
    rng = np.random.default_rng(seed)
    cnt = rng.poisson(scale, size=(M, El)) if scale else np.zeros((M, El), dtype=int)
    # one minibatch always fits in the ring (the entry point refuses smaller rings)
    cnt = np.minimum(cnt, (ring // El) // 128 * 128 - 1)
    plan = O.stream_plan(cnt, ring, min_rows)
    pad = lambda c: int(np.sum((np.asarray(c) + 127) // 128 * 128))
    # consecutive minibatch ranges covering [0, M)
    ends = [b for _, b in plan["macro"]]
    starts = [a for a, _ in plan["macro"]]
    assert starts[0] == 0 and ends[-1] == M and starts[1:] == ends[:-1]
    for i, (a, b) in enumerate(plan["macro"]):
        rows = pad(cnt[a:b].sum(0))
        assert rows == plan["sizes"][i] <= ring
        if b < M:  # closed early: two waves reached, or the next minibatch would not fit
            assert rows >= min_rows or pad(cnt[a:b + 1].sum(0)) > ring
        if b - a > 1:  # it did not reach two waves before its last minibatch
            assert pad(cnt[a:b - 1].sum(0)) < min_rows
    assert plan["resident"] == _simulate(plan, ring)
    # the chunks walk the macrobatches in reverse, each fitting in the ring
    covered = []
    for lo, hi in plan["chunks"]:
        covered = list(range(lo, hi)) + covered
        assert sum(plan["sizes"][lo:hi]) <= ring
    assert covered == list(range(len(plan["macro"]))) or plan["chunks"] == [(0, 0)]
    first = plan["chunks"][0]
    assert all(plan["resident"][m] for m in range(*first)) or first[1] - first[0] <= 1
    assert plan["replayed"] == sum(s for m, s in enumerate(plan["sizes"]) if not (first[0] <= m < first[1]
                                                                                    and plan["resident"][m]))
    assert plan["rows"] == sum(plan["sizes"])
