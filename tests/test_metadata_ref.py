"""Pins of the split-KV scheduling reference (CPU only)."""
import numpy as np
import pytest

from oracle import metadata_ref as M


def test_hand_worked_example():
    """tiles [2, 1] over 2 partitions: costs [7, 6], T = 13, boundaries at
    cost positions 0, 6, 13 -> (0,0), (0,1), (2,0)."""
    md, ns = M.schedule([2, 1], 2)
    assert ns == [0, 2, 3]
    assert md[0] == [0, 0, 0, 1, 0, 0, 0, 0]
    assert md[1] == [0, 1, 2, 0, 1, 0, 0, 0]


def test_hand_worked_example_with_empty_unit_and_spare_partitions():
    """tiles [0, 1, 0] over 4 partitions: costs [0, 6, 0], T = 6, positions
    0, 1, 3, 4, 6 all fall in the overhead of unit 1 (page 0) except the end."""
    md, ns = M.schedule([0, 1, 0], 4)
    assert ns == [0, 0, 1, 1]
    assert [r[:5] for r in md] == [[1, 0, 1, 0, 0], [1, 0, 1, 0, 0], [1, 0, 1, 0, 0], [1, 0, 3, 0, 0]]


def _check_plan(tiles, num_parts):
    md, ns = M.schedule(tiles, num_parts)
    U = len(tiles)
    assert len(md) == num_parts and len(ns) == U + 1
    # every (unit, page) covered exactly once, in order
    seen = []
    split_of = {}
    next_id = {}
    for p, row in enumerate(md):
        segs = M.segments(row, tiles)
        for k, (u, a, b) in enumerate(segs):
            seen.extend((u, j) for j in range(a, b))
            sid = row[4] if k == 0 else ns[u]
            if a == 0:
                assert sid == ns[u]
            else:
                assert sid == next_id[u]
            split_of[(u, a)] = sid
            next_id[u] = sid + 1
        # load bound: pages + fixed cost per segment <= ceil(T/P) + FIXED
        load = sum(b - a + M.FIXED_COST for (u, a, b) in segs)
        total = sum(n + M.FIXED_COST for n in tiles if n > 0)
        assert load <= -(-total // num_parts) + 2 * M.FIXED_COST
    expect = [(u, j) for u in range(U) for j in range(tiles[u])]
    assert seen == expect
    # split counts match num_splits; contiguous ids per unit
    for u in range(U):
        n_split = ns[u + 1] - ns[u]
        ids = sorted(v for (uu, a), v in split_of.items() if uu == u)
        assert len(ids) == n_split
        assert ids == list(range(ns[u], ns[u + 1]))
        assert (n_split >= 1) == (tiles[u] > 0)
    assert all(a <= b for a, b in zip(ns, ns[1:]))
    return md, ns


@pytest.mark.parametrize("seed", range(12))
def test_plan_invariants_random(seed):
    rng = np.random.default_rng(seed)
    U = int(rng.integers(1, 80))
    lens = rng.integers(0, 9000, size=U)
    lens[rng.random(U) < 0.1] = 0
    tiles = M.unit_tiles(lens)
    for P in (1, 2, 7, 74, 148, 592):
        _check_plan(tiles, P)


def test_plan_single_long_sequence_spreads_over_all_parts():
    md, ns = _check_plan(M.unit_tiles([32768]), 148)
    assert ns[1] == len({tuple(r[:2]) for r in md})      # one split per distinct start
    assert ns[1] > 100


def test_sparse_units():
    tiles = M.unit_tiles([5, 9], s_q=2, topk=130)
    assert tiles == [3, 3, 3, 3]
    _check_plan(tiles, 5)


def test_all_empty():
    md, ns = M.schedule([0, 0], 3)
    assert ns == [0, 0, 0]
    assert all(r[:5] == [2, 0, 2, 0, 0] for r in md)
