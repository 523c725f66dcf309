"""Plain-Python restatement of the db-SP work partition (test infrastructure only).

"db-SP: ... Sparsity-Aware Sequence Parallelism ..." (abstract) balances block-sparse attention over
sequence-parallel ranks by a dual-level partition (heads, then blocks) and measures balance with a sparse
imbalance ratio; the page gives neither formula nor algorithm.  This file states the reading the library
implements, step by step and with loops, so that its output can be compared with the library's exactly:

  unit (h, qp): head h, query tiles 2qp and 2qp+1 (qp < NP = ceil(T/2)); cost = tiles its rows keep
  (keys j <= i when causal);
  imbalance ratio = max rank load / mean rank load;
  level 1: heads in decreasing total cost (ties: lower head), each to the least loaded rank (ties: lower);
  level 2: repeat: M = most loaded rank, m = least loaded (ties: lower rank), gap = load(M) - load(m); among
  M's units with 0 < cost < gap take the one minimising |2 cost - gap| (ties: larger cost, then the lower
  unit index h * NP + qp) and give it to m; stop when there is none.

Only the tests may import this module.  It shares no code with the library.  Pinned in
tests/test_dbsp_plan.py (closed forms for dense masks, invariants, brute-force optimum on small cases).
"""
from __future__ import annotations

import numpy as np


def unit_costs(block_mask, H: int, T: int, causal: bool):
    """cost[h][qp] = number of kept tiles (h, i, j) with i in {2qp, 2qp+1}, i < T, j < T, and j <= i if causal.
    block_mask None means every tile is kept."""
    NP = (T + 1) // 2
    cost = [[0] * NP for _ in range(H)]
    for h in range(H):
        for qp in range(NP):
            c = 0
            for i in (2 * qp, 2 * qp + 1):
                if i >= T:
                    continue
                for j in range(T):
                    if causal and j > i:
                        continue
                    if block_mask is None or block_mask[h][i][j] != 0:
                        c += 1
            cost[h][qp] = c
    return cost


def imbalance(loads) -> float:
    total = sum(loads)
    return max(loads) * len(loads) / total if total > 0 else 1.0


def plan(cost, P: int):
    """Returns (unit_rank[h][qp], loads[P])."""
    H, NP = len(cost), len(cost[0])
    loads = [0] * P
    rank = [[-1] * NP for _ in range(H)]
    head_total = [sum(cost[h]) for h in range(H)]
    heads = sorted(range(H), key=lambda h: (-head_total[h], h))
    for h in heads:  # level 1
        r = min(range(P), key=lambda x: (loads[x], x))
        for qp in range(NP):
            rank[h][qp] = r
        loads[r] += head_total[h]
    while True:  # level 2
        M = min(range(P), key=lambda x: (-loads[x], x))
        m = min(range(P), key=lambda x: (loads[x], x))
        gap = loads[M] - loads[m]
        best = None
        for h in range(H):
            for qp in range(NP):
                c = cost[h][qp]
                if rank[h][qp] != M or not (0 < c < gap):
                    continue
                key = (abs(2 * c - gap), -c, h * NP + qp)
                if best is None or key < best[0]:
                    best = (key, h, qp, c)
        if best is None:
            break
        _, h, qp, c = best
        rank[h][qp] = m
        loads[M] -= c
        loads[m] += c
    return rank, loads


def rank_items(cost, rank, B: int, r: int):
    """Kernel item ids (b * H + h) * NP + qp of rank r: units by decreasing cost (ties: lower unit index),
    each for b = 0 .. B-1."""
    H, NP = len(cost), len(cost[0])
    units = [(h, qp) for h in range(H) for qp in range(NP) if rank[h][qp] == r]
    units.sort(key=lambda u: (-cost[u[0]][u[1]], u[0] * NP + u[1]))
    return [(b * H + h) * NP + qp for (h, qp) in units for b in range(B)]


def as_lists(mask_np):
    return None if mask_np is None else np.asarray(mask_np).tolist()
