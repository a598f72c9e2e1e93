"""Host-side placement of the peer-memory transport of expert parallelism
(mixture_experts_feed_b200.ep.p2p_tables), checked by placing every row of
every rank one by one: each permuted row of each source lands on its own row
of its owner's receive buffer, the receive buffer is ordered by (local
expert, source, row), and the return mapping sends every received row back
to the permuted row it came from.  CPU only."""
from __future__ import annotations

import random

import pytest

from mixture_experts_feed_b200.ep import p2p_tables


def random_offsets(rng, E, T, k, empty_frac):
    counts = [0 if rng.random() < empty_frac else rng.randint(0, 3 * T * k // E + 1) for _ in range(E)]
    off = [0]
    for c in counts:
        off.append(off[-1] + c)
    return off


def expert_of(off, i):
    e = 0
    while off[e + 1] <= i:
        e += 1
    return e


@pytest.mark.parametrize("W,El,seed", [(1, 8, 0), (2, 4, 1), (4, 3, 2), (8, 2, 3), (3, 5, 4)])
def test_rows_land_once_in_order_and_come_back(W, El, seed):
    rng = random.Random(seed)
    E = W * El
    offsets = [random_offsets(rng, E, 40, 3, 0.3) for _ in range(W)]
    tabs = [p2p_tables(offsets, r, El) for r in range(W)]
    assert len({t["max_rows_in"] for t in tabs}) == 1
    recv = [[None] * tabs[d]["rows_in"] for d in range(W)]
    for s in range(W):
        off = offsets[s]
        for i in range(off[E]):
            e = expert_of(off, i)
            d = e // El
            row = tabs[s]["dst_base"][e] + i - off[e]
            assert 0 <= row < tabs[d]["rows_in"], (s, i, row)
            assert recv[d][row] is None, f"two rows at receiver {d} row {row}"
            recv[d][row] = (e % El, s, i)
    for d in range(W):
        assert all(v is not None for v in recv[d])
        assert recv[d] == sorted(recv[d])                 # local expert, then source, then row
        t = tabs[d]
        assert t["run_start"][0] == 0 and t["run_start"][-1] == t["rows_in"]
        assert t["loc"][-1] == t["rows_in"] and len(t["loc"]) == El + 1
        for j, (el, s, i) in enumerate(recv[d]):
            run = max(q for q in range(E) if t["run_start"][q] <= j)
            assert divmod(run, W) == (el, s)
            assert t["src_base"][run] + j - t["run_start"][run] == i
            assert t["loc"][el] <= j < t["loc"][el + 1]


def test_a_misplaced_run_is_caught():
    """The brute-force check above fails when the sources' runs are not
    staggered (a planted mistake: every source's run of an expert starting at
    the expert's first row)."""
    W, El = 2, 2
    offsets = [[0, 2, 3, 5, 6], [0, 1, 3, 3, 4]]
    tabs = [p2p_tables(offsets, r, El) for r in range(W)]
    bad = [dict(t, dst_base=[tabs[0]["dst_base"][e] for e in range(W * El)]) for t in tabs]
    seen = set()
    clash = False
    for s in range(W):
        off = offsets[s]
        for i in range(off[-1]):
            e = expert_of(off, i)
            key = (e // El, bad[s]["dst_base"][e] + i - off[e])
            clash |= key in seen
            seen.add(key)
    assert clash
