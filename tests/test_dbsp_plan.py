"""The db-SP work partition: the plain-Python oracle pinned to hand-worked examples, closed forms,
invariants and brute force; then the library's planner (C++, through the C ABI, host only) against it,
exactly."""
import itertools
import json
import os

import numpy as np
import pytest

import oracle.dbsp_plan as op
from sequence_head_attention_b200 import spattn, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dbsp_plan_examples.json")


def _random_mask(H, T, seed, p_lo=0.1, p_hi=0.9):
    rng = np.random.default_rng(seed)
    p = rng.uniform(p_lo, p_hi, size=H)
    m = (rng.random((H, T, T)) < p[:, None, None]).astype(np.uint8)
    for h in range(H):
        np.fill_diagonal(m[h], 1)
    return m


# --- oracle pins ------------------------------------------------------------------------------------
def test_oracle_plan_matches_hand_worked_examples():
    for e in json.load(open(GOLDEN))["examples"]:
        rank, loads = op.plan(e["cost"], e["P"])
        assert rank == e["unit_rank"], e["notes"]
        assert loads == e["loads"]
        assert op.imbalance(loads) == pytest.approx(e["imbalance"], rel=1e-12)


@pytest.mark.parametrize("T", [1, 2, 7, 8])
def test_oracle_costs_closed_forms(T):
    NP = (T + 1) // 2
    dense = op.unit_costs(None, 2, T, causal=False)
    causal = op.unit_costs(None, 2, T, causal=True)
    for qp in range(NP):
        rows = [i for i in (2 * qp, 2 * qp + 1) if i < T]
        assert dense[1][qp] == len(rows) * T           # every tile of the unit's rows
        assert causal[1][qp] == sum(i + 1 for i in rows)  # row i keeps keys 0..i
    assert sum(map(sum, causal)) == 2 * T * (T + 1) // 2


def test_oracle_costs_count_kept_tiles():
    H, T = 3, 9
    m = _random_mask(H, T, seed=5)
    for causal in (False, True):
        cost = op.unit_costs(m.tolist(), H, T, causal)
        keep = np.tril(m) if causal else m
        per_row = keep.sum(axis=2)  # [H, T]
        for h in range(H):
            for qp in range((T + 1) // 2):
                assert cost[h][qp] == per_row[h, 2 * qp:2 * qp + 2].sum()
    one = np.zeros((H, T, T), dtype=np.uint8)
    one[2, 5, 3] = 1
    cost = op.unit_costs(one.tolist(), H, T, False)
    assert sum(map(sum, cost)) == 1 and cost[2][2] == 1


@pytest.mark.parametrize("seed", range(6))
def test_oracle_plan_invariants_and_brute_force_bound(seed):
    rng = np.random.default_rng(seed)
    H, NP, P = int(rng.integers(1, 4)), int(rng.integers(1, 4)), int(rng.integers(2, 4))
    cost = rng.integers(0, 9, size=(H, NP)).tolist()
    rank, loads = op.plan(cost, P)
    # every unit on exactly one valid rank; loads are the sums of their units
    assert all(0 <= rank[h][q] < P for h in range(H) for q in range(NP))
    recount = [sum(cost[h][q] for h in range(H) for q in range(NP) if rank[h][q] == r) for r in range(P)]
    assert recount == loads and sum(loads) == sum(map(sum, cost))
    # stopping rule: no unit of the most loaded rank could lower the spread
    M = max(range(P), key=lambda r: (loads[r], -r))
    gap = max(loads) - min(loads)
    assert not any(rank[h][q] == M and 0 < cost[h][q] < gap for h in range(H) for q in range(NP))
    # the result is within the largest unit of the best possible partition (found by brute force)
    units = [cost[h][q] for h in range(H) for q in range(NP)]
    best = min(max(sum(c for c, a in zip(units, asg) if a == r) for r in range(P))
               for asg in itertools.product(range(P), repeat=len(units)))
    assert max(loads) <= best + max(units)
    assert max(loads) >= best


def test_oracle_level_two_never_raises_the_head_level_maximum():
    rng = np.random.default_rng(3)
    for _ in range(20):
        H, NP, P = 5, 4, 3
        cost = rng.integers(0, 20, size=(H, NP)).tolist()
        totals = sorted(((sum(cost[h]), h) for h in range(H)), key=lambda x: (-x[0], x[1]))
        level1 = [0] * P
        for tot, _h in totals:
            r = min(range(P), key=lambda x: (level1[x], x))
            level1[r] += tot
        _, loads = op.plan(cost, P)
        assert max(loads) <= max(level1)


# --- library against the oracle ----------------------------------------------------------------------
@pytest.mark.parametrize("H,T,P,causal,seed", [
    (4, 8, 2, False, 0), (5, 9, 3, True, 1), (8, 16, 4, False, 2), (8, 16, 4, True, 3), (3, 1, 2, False, 4),
    (6, 11, 5, True, 5),
])
def test_library_plan_equals_oracle(H, T, P, causal, seed):
    m = _random_mask(H, T, seed)
    cost_lib = spattn.sp_dbsp_unit_costs(m, H, T, causal)
    cost_orc = op.unit_costs(m.tolist(), H, T, causal)
    assert cost_lib.tolist() == cost_orc
    rank_lib, load_lib, imb_lib = spattn.sp_dbsp_plan(cost_lib, P)
    rank_orc, load_orc = op.plan(cost_orc, P)
    assert rank_lib.tolist() == rank_orc
    assert load_lib.tolist() == load_orc
    assert imb_lib == pytest.approx(op.imbalance(load_orc), rel=1e-12)
    for B in (1, 2):
        for r in range(P):
            assert spattn.sp_dbsp_rank_items(cost_lib, rank_lib, B, r).tolist() == op.rank_items(cost_orc, rank_orc, B, r)


def test_library_plan_on_the_block_sparse_workload_mask():
    """The 40-head, 256-tile mask of the block-sparse workload over 4 ranks: same plan as the oracle, and
    better balanced than the contiguous head split of Ulysses."""
    w = synth.WORKLOADS["block_sparse"]
    mask = synth.block_mask(w.H, w.S, seed=0).numpy()
    T = mask.shape[-1]
    cost = spattn.sp_dbsp_unit_costs(mask, w.H, T, False)
    rank, load, imb = spattn.sp_dbsp_plan(cost, 4)
    rank_orc, load_orc = op.plan(cost.tolist(), 4)
    assert rank.tolist() == rank_orc and load.tolist() == load_orc
    head_split = [int(cost[r * w.H // 4:(r + 1) * w.H // 4].sum()) for r in range(4)]
    assert imb < op.imbalance(head_split)
    assert imb <= 1.0 + cost.max() * 4 / cost.sum()


def test_library_rejects_bad_arguments():
    with pytest.raises(spattn.SpError):
        spattn.sp_dbsp_plan(np.zeros((2, 2), dtype=np.int64), 0)
    with pytest.raises(spattn.SpError):
        spattn.sp_dbsp_plan(-np.ones((2, 2), dtype=np.int64), 2)
