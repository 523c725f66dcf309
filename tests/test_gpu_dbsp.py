"""Per-rank attention over planned work-item lists (sp_attn_fwd_items): the ranks' launches together write
exactly what one launch writes (bitwise: each item's arithmetic is the same), which matches the oracle."""
import pytest
import torch

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


def _ranks_launch(q, k, v, cost, unit_rank, P, causal, mask):
    B, S, H, D = q.shape
    o = torch.full((B, S, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, S), float("nan"), device="cuda")
    for r in range(P):
        items = torch.from_numpy(spattn.sp_dbsp_rank_items(cost, unit_rank, B, r)).cuda()
        spattn.sp_attn_fwd_items(q, k, v, o, lse, items, causal=causal, block_mask=mask)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    return o, lse


@pytest.mark.parametrize("B,S,H,D,P,causal,sparse", [
    (1, 2048, 8, 128, 4, False, True), (2, 1000, 3, 64, 2, True, True), (1, 1536, 6, 128, 3, True, False),
])
def test_planned_ranks_equal_one_launch_and_oracle(B, S, H, D, P, causal, sparse):
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=S + P, scale=0.5))
    T = (S + 127) // 128
    mask_cpu = synth.block_mask(H, S, seed=P) if sparse else None
    mask = None if mask_cpu is None else mask_cpu.cuda()
    cost = spattn.sp_dbsp_unit_costs(mask_cpu, H, T, causal)
    unit_rank, _, _ = spattn.sp_dbsp_plan(cost, P)
    o, lse = _ranks_launch(q, k, v, cost, unit_rank, P, causal, mask)
    o1 = torch.empty_like(o)
    l1 = torch.empty_like(lse)
    spattn.sp_attn_fwd(q, k, v, o1, l1, causal=causal, block_mask=mask)
    torch.cuda.synchronize()
    assert torch.equal(o, o1) and torch.equal(lse, l1)
    ref = oracle.attention(to64(q.cpu()), to64(k.cpu()), to64(v.cpu()), causal=causal,
                           block_mask=None if mask_cpu is None else mask_cpu.numpy())
    assert_close(o, ref[0], lse, ref[1])


def test_unknown_item_is_skipped_and_reported():
    B, S, H, D = 1, 1024, 2, 128
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=3, scale=0.5))
    NP = (S // 128 + 1) // 2
    o = torch.full((B, S, H, D), 5.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, S), 5.0, device="cuda")
    items = torch.tensor([3, B * H * NP, 0], dtype=torch.int32, device="cuda")  # the middle id does not exist
    spattn.sp_attn_fwd_items(q, k, v, o, lse, items)
    assert spattn.sp_check_device_error() == spattn.SP_ERR_INVALID_ARG
    assert spattn.sp_check_device_error() == spattn.SP_OK  # cleared
    ref = oracle.attention(to64(q.cpu()), to64(k.cpu()), to64(v.cpu()))
    # item 0: head 0, rows 0-255; item 3: head 0, rows 768-1023 (NP = 4)
    for rows in (slice(0, 256), slice(768, 1024)):
        assert_close(o[:, rows, 0:1], ref[0][:, rows, 0:1], lse[:, 0:1, rows], ref[1][:, 0:1, rows])
    assert torch.all(o[:, 256:768, 0] == 5.0) and torch.all(o[:, :, 1] == 5.0)
    assert torch.all(lse[:, 1] == 5.0)


def test_empty_item_list_is_a_no_op():
    q = torch.zeros((1, 256, 1, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 2.0)
    spattn.sp_attn_fwd_items(q, q, q, o, None, torch.zeros(0, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.all(o == 2.0)


@pytest.mark.parametrize("causal", [False, True])
def test_masked_launch_in_cost_order_equals_natural_order(causal):
    """sp_attn_fwd with a mask claims its items in its cost order; the result is bitwise that of the
    same items claimed in their natural order (each item's arithmetic does not depend on the order)."""
    B, S, H, D = 2, 3000, 5, 128
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=77, scale=0.5))
    mask = synth.block_mask(H, S, seed=77).cuda()
    T = (S + 127) // 128
    NP = (T + 1) // 2
    o1 = torch.empty_like(q)
    l1 = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd(q, k, v, o1, l1, causal=causal, block_mask=mask)
    items = torch.arange(B * H * NP, dtype=torch.int32, device="cuda")
    o2 = torch.full_like(q, float("nan"))
    l2 = torch.full((B, H, S), float("nan"), device="cuda")
    spattn.sp_attn_fwd_items(q, k, v, o2, l2, items, causal=causal, block_mask=mask)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_masked_launch_work_order_heads_densest_first_items_longest_first():
    """The work order a masked sp_attn_fwd writes into its workspace (the last section: B * H * ceil(T / 2)
    item ids) is a permutation of the items that keeps each (b, h)'s items together, takes the (b, h) in
    order of their head's kept tiles, most first (ties: lower b * H + h first), and within a (b, h) runs from
    the item with the most kept tiles to the fewest (cost of item (b, h, qp) = kept tiles of query-tile rows
    2 qp and 2 qp + 1 of head h's mask)."""
    B, S, H, D = 2, 3000, 5, 128
    T = (S + 127) // 128
    NP = (T + 1) // 2
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=78, scale=0.5))
    mask = synth.block_mask(H, S, seed=78)
    ws_bytes = spattn.sp_attn_fwd_workspace_bytes(B, S, H, D, 1, True)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd(q, k, v, o, lse, block_mask=mask.cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    n = B * H * NP
    off = ws_bytes - (n * 4 + 255) // 256 * 256
    order = ws[off:off + 4 * n].cpu().view(torch.int32).numpy()
    assert sorted(order.tolist()) == list(range(n))
    rows = (mask != 0).sum(dim=2).numpy()  # kept tiles per (head, query-tile row)
    total = rows.sum(axis=1)
    segs = sorted(range(B * H), key=lambda sg: (-int(total[sg % H]), sg))
    assert len(set(total.tolist())) > 1  # the heads' order is not the natural one by accident
    for r, seg in enumerate(segs):
        ids = order[r * NP:(r + 1) * NP]
        assert set((ids // NP).tolist()) == {seg}
        h = seg % H
        cost = [int(rows[h, 2 * qp]) + (int(rows[h, 2 * qp + 1]) if 2 * qp + 1 < T else 0) for qp in ids % NP]
        assert all(a >= b for a, b in zip(cost, cost[1:])), cost
