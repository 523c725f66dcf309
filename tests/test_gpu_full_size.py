"""The full-size workloads, in the launch configuration the benchmark times, checked on sampled query
rows against the oracle (which evaluates those rows one by one over all keys)."""
import pytest
import torch

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import spattn, synth
from sequence_head_attention_b200 import workloads

pytestmark = pytest.mark.gpu
N_ROWS = 96


def _oracle_rows(q, k, v, rows, **kw):
    return oracle.attention(to64(q), to64(k), to64(v), rows=rows, **kw)


def _sampled(o, lse, rows):
    r = torch.tensor(rows, device=o.device)
    return o[:, r], lse[:, :, r]


def test_video_dit_ulysses_step():
    w = synth.WORKLOADS["video_dit"]
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=0, scale=w.scale)
    sr = w.S // w.ranks  # rows per sequence shard: each shard's first and last rows, and its short last tile
    rows = synth.sample_rows(w.S, N_ROWS, seed=0,
                             must=[x for r in range(w.ranks) for x in (r * sr, r * sr + 63 * 128, (r + 1) * sr - 1)])
    ref = _oracle_rows(q, k, v, rows)
    # attention on the full 40-head tensors with the uneven head chunks
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.S), device="cuda")
    spattn.sp_attn_fwd(qd, kd, vd, o, lse, head_chunks=list(w.head_chunks))
    assert spattn.sp_check_device_error() == spattn.SP_OK
    o_s, l_s = _sampled(o, lse, rows)
    assert_close(o_s, ref[0], l_s, ref[1])
    # the Ulysses step the benchmark times: seq shards -> head shards -> per-rank attention -> back
    step = workloads.UlyssesStep(w, q, k, v)
    step.run()
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    o_full = torch.cat(step.o_seq, dim=1)
    assert torch.equal(o_full, o)  # same per-head arithmetic, bitwise
    lse_full = step.lse_full()
    assert torch.equal(lse_full, lse)
    # the same step with the relayouts folded into the attention kernel (shards of 8190 rows, tiled on
    # their own grids: 63 full tiles and one of 126 rows each)
    fused = workloads.UlyssesStep(w, q, k, v, fused=True)
    fused.run()
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    o_fused = torch.cat(fused.o_seq, dim=1)
    o_s, l_s = _sampled(o_fused, fused.lse_full(), rows)
    assert_close(o_s, ref[0], l_s, ref[1])
    assert_close(o_fused, o, fused.lse_full(), lse)


def test_ring_causal_partials_and_merge():
    """The ring step the benchmark times (8 KV blocks of 7168: the first block's partial, seven blocks merged
    in place, the running O rounded to bf16), the standalone re-merge of the 8 materialised partials, and
    sp_attn_fwd with n_kv_blocks = 8: each checked on sampled rows against the oracle."""
    w = synth.WORKLOADS["ring_causal"]
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=0, scale=w.scale)
    blk = w.S // w.n_kv_blocks
    rows = synth.sample_rows(w.S, N_ROWS, seed=1, must=[blk - 1, blk, 4 * blk, 4 * blk - 1, w.S - blk])
    ref = _oracle_rows(q, k, v, rows, causal=True)
    step = workloads.RingStep(w, q, k, v, with_partials=True)
    step.run()
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    o_s, l_s = _sampled(step.o, step.lse, rows)
    assert_close(o_s, ref[0], l_s, ref[1])
    step.partials()
    step.merge()
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    o_s, l_s = _sampled(step.o_merged, step.lse_merged, rows)
    assert_close(o_s, ref[0], l_s, ref[1])
    # one call with n_kv_blocks = 8 does the same partials and merge
    o2 = torch.empty_like(step.o)
    l2 = torch.empty_like(step.lse)
    del step.o_parts, step.l_parts
    spattn.sp_attn_fwd(step.q, step.k, step.v, o2, l2, n_kv_blocks=w.n_kv_blocks, causal=True,
                       workspace=step.workspace_for_fwd())
    assert torch.equal(o2, step.o_merged) and torch.equal(l2, step.lse_merged)


def test_block_sparse_dit():
    w = synth.WORKLOADS["block_sparse"]
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=0, scale=w.scale)
    mask = synth.block_mask(w.H, w.S, seed=0)
    T = mask.shape[-1]
    rows = synth.sample_rows(w.S, N_ROWS, seed=2, must=[128 * t + 3 for t in range(0, T, 9)])
    ref = _oracle_rows(q, k, v, rows, block_mask=mask.numpy())
    step = workloads.SparseStep(w, q, k, v, mask)
    step.run()
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    o_s, l_s = _sampled(step.o, step.lse, rows)
    assert_close(o_s, ref[0], l_s, ref[1])
    # the db-SP launches the benchmark times: four simulated ranks' planned item lists write exactly what
    # the single launch wrote (each item's arithmetic is the same)
    o1, l1 = step.o.clone(), step.lse.clone()
    step.o.fill_(float("nan"))
    step.lse.fill_(float("nan"))
    lists, imb = step.rank_items(4, planned=True)
    for items in lists:
        step.run_items(items)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    assert imb < 1.01
    assert torch.equal(step.o, o1) and torch.equal(step.lse, l1)


def test_video_dit_rank_backward():
    """The backward the benchmark times (sp_attn_bwd on one simulated rank's 10 heads of video_dit, dense,
    B1 S32760 D128), checked on sampled query rows (dq) and key rows (dk, dv) of one head against the
    oracle, which evaluates each sampled row over all keys or queries.  Tolerance as in
    tests/test_gpu_attn_bwd.py (rel-L2 1e-2, max-abs 2e-2 of the largest reference value)."""
    import numpy as np
    w = synth.WORKLOADS["video_dit"]
    hl = w.H // w.ranks
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=0, scale=w.scale)
    q, k, v = (t[:, :, :hl].contiguous() for t in (q, k, v))
    do = torch.randn(q.shape, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, hl, w.S), device="cuda")
    spattn.sp_attn_fwd(qd, kd, vd, o, lse)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    spattn.sp_attn_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    rows = synth.sample_rows(w.S, 32, seed=5, must=[127, 128, 16383, 16384])
    heads = [hl // 2]
    rq, rk, rv = oracle.attention_bwd_rows(to64(q), to64(k), to64(v), to64(do), heads=heads, q_rows=rows,
                                           k_rows=rows)
    r = torch.tensor(rows)
    for x, ref, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")):
        got = to64(x.cpu()[:, r][:, :, heads])
        d = got - ref
        rel = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-3 * np.sqrt(ref.size))
        mx = np.max(np.abs(d)) / max(np.max(np.abs(ref)), 1e-3)
        assert np.all(np.isfinite(got)), name
        assert rel <= 1e-2 and mx <= 2e-2, (name, rel, mx)
