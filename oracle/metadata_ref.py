"""Split-KV scheduling plan, restated sequentially in plain Python.

Test infrastructure only (see the package docstring).

The pages show the call ``tile_scheduler_metadata, num_splits =
get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv)``, made once before
the per-layer decode loop ("Was ist FlashMLA?" (topnet.top), section
"2. MLA-Metadaten abrufen"), but not the algorithm behind it.  The plan below
is this project's own; its constants are part of the contract.

Work units and costs
    A unit is one sequence (dense path) or one (sequence, query token) pair
    (sparse path).  Unit u has n_u work tiles: ceil(L_u / 64) cache pages on
    the dense path, ceil(topk / 64) index tiles on the sparse path.  Its cost
    is c_u = n_u + FIXED_COST when n_u > 0, else 0 (FIXED_COST models the
    per-split query load, epilogue and combine, in page-equivalents).
Partition boundaries
    With C_u the exclusive prefix sum of the costs and T their total, boundary
    p (0 <= p <= P) sits at cost position x_p = floor(p * T / P).  A position
    x < T lies in the unit u with C_u <= x < C_u + c_u, at page
    j = max(0, x - C_u - FIXED_COST); x = T maps to (U, 0).
    Partition p covers the (unit, page) pairs from boundary p (inclusive) to
    boundary p + 1 (exclusive), in batch order.
Splits
    A non-empty unit has 1 + (number of distinct boundary points (u, j) with
    j > 0) splits.  num_splits[u] is the exclusive prefix sum of the split
    counts (length U + 1).  A partition's first segment has split index
    num_splits[u_p] + (number of distinct boundary points (u_p, j) with
    0 < j <= j_p).
Output
    tile_md[p] = (u_p, j_p, u_{p+1}, j_{p+1}, first_split_idx_p, 0, 0, 0).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

PAGE = 64
FIXED_COST = 5
MD_WORDS = 8


def unit_tiles(cache_seqlens: Sequence[int], s_q: int = 1, topk: int = 0) -> List[int]:
    """Work tiles per unit: pages per sequence (dense) or, for the sparse
    path, ceil(topk / 64) per (sequence, token) unit."""
    if topk > 0:
        per = (topk + PAGE - 1) // PAGE
        return [per for _ in cache_seqlens for _ in range(s_q)]
    return [(int(L) + PAGE - 1) // PAGE if int(L) > 0 else 0 for L in cache_seqlens]


def schedule(tiles: Sequence[int], num_parts: int) -> Tuple[List[List[int]], List[int]]:
    """Plan for units with ``tiles`` work tiles over ``num_parts`` partitions.
    Returns (tile_md [num_parts][8], num_splits [U + 1])."""
    U = len(tiles)
    costs = [n + FIXED_COST if n > 0 else 0 for n in tiles]
    starts = []
    acc = 0
    for c in costs:
        starts.append(acc)
        acc += c
    total = acc

    def locate(x: int) -> Tuple[int, int]:
        if x >= total:
            return (U, 0)
        for u in range(U):
            if starts[u] <= x < starts[u] + costs[u]:
                return (u, max(0, x - starts[u] - FIXED_COST))
        raise AssertionError("position outside every unit")

    bounds = [locate((p * total) // num_parts) for p in range(num_parts + 1)]

    # distinct interior cut points per unit
    cuts = [set() for _ in range(U)]
    for (u, j) in bounds:
        if u < U and j > 0:
            cuts[u].add(j)
    splits = [(1 + len(cuts[u])) if tiles[u] > 0 else 0 for u in range(U)]
    num_splits = [0]
    for s in splits:
        num_splits.append(num_splits[-1] + s)

    tile_md = []
    for p in range(num_parts):
        (u0, j0), (u1, j1) = bounds[p], bounds[p + 1]
        if u0 >= U:
            first = num_splits[U]
        else:
            first = num_splits[u0] + sum(1 for j in cuts[u0] if 0 < j <= j0)
        tile_md.append([u0, j0, u1, j1, first, 0, 0, 0])
    return tile_md, num_splits


def segments(tile_md_row: Sequence[int], tiles: Sequence[int]):
    """The (unit, first page, end page) segments partition ``tile_md_row``
    covers, in order."""
    u0, j0, u1, j1 = tile_md_row[:4]
    out = []
    u, j = u0, j0
    while (u, j) < (u1, j1) and u < len(tiles):
        end = tiles[u] if u < u1 else j1
        if end > j:
            out.append((u, j, end))
        u, j = u + 1, 0
    return out
