"""Attention straight on the Ulysses sequence shards (sp_attn_fwd_seq_sharded) against the relayout
path it replaces and against the fp64 oracle.

Shard lengths that are and are not multiples of the 128-row tile.  The kernel lays query and key tiles on
each shard's own grid: with S/P a multiple of 128 that is the global grid and the result equals the
relayout path bit for bit; otherwise each shard ends in a short tile (shards shorter than one tile are a
single short tile) and the result equals it within the parity tolerance."""
import pytest
import torch

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import spattn, synth
from sequence_head_attention_b200.workloads import rank_chunks

pytestmark = pytest.mark.gpu


def relayout_path(qs, ks, vs, P, H, chunks, causal):
    """seq -> head relayout, per-rank sp_attn_fwd, head -> seq relayout (the unfused Ulysses step)."""
    B, Sl, _, D = qs[0].shape
    S, Hl = Sl * P, H // P
    heads = [[torch.empty((B, S, Hl, D), dtype=torch.bfloat16, device="cuda") for _ in range(P)] for _ in range(4)]
    spattn.sp_seq_to_head_relayout(qs, heads[0])
    spattn.sp_seq_to_head_relayout(ks, heads[1])
    spattn.sp_seq_to_head_relayout(vs, heads[2])
    lse = []
    for r in range(P):
        l_r = torch.empty((B, Hl, S), device="cuda")
        spattn.sp_attn_fwd(heads[0][r], heads[1][r], heads[2][r], heads[3][r], l_r, head_chunks=chunks[r],
                           causal=causal)
        lse.append(l_r)
    o_seq = [torch.empty_like(qs[0]) for _ in range(P)]
    spattn.sp_head_to_seq_relayout(heads[3], o_seq)
    return o_seq, torch.cat(lse, dim=1)


def fused_path(qs, ks, vs, P, H, chunks, causal):
    B, Sl, _, D = qs[0].shape
    Hl = H // P
    o_seq = [torch.full_like(qs[0], float("nan")) for _ in range(P)]
    lse = torch.full((B, H, Sl * P), float("nan"), device="cuda")
    for r in range(P):
        spattn.sp_attn_fwd_seq_sharded(qs, ks, vs, o_seq, lse, heads=(r * Hl, Hl), head_chunks=chunks[r],
                                       causal=causal)
    return o_seq, lse


@pytest.mark.parametrize("B,S,H,D,P,chunks,causal", [
    (1, 1000, 4, 128, 4, None, False),      # shards of 250 rows: two tiles per shard, the second short
    (1, 1000, 8, 128, 8, [3, 5], True),     # shards of 125 rows: one short tile per shard
    (2, 1024, 4, 64, 4, [1, 3], False),     # shards of 256 rows: the global grid
    (1, 2046, 6, 128, 3, [2, 4], True),     # shards of 682 rows: 6 tiles each, the last short
    (1, 1536, 2, 64, 2, None, True),        # shards of 768 rows: the global grid
    (1, 1280, 2, 128, 2, None, True),       # shards of 640 rows: 5 tiles each, an odd count
])
def test_fused_equals_relayout_path_and_oracle(B, S, H, D, P, chunks, causal):
    q, k, v = synth.qkv(B, S, H, D, seed=S + P, scale=0.5)
    qs = [t.cuda() for t in synth.split_seq(q, P)]
    ks = [t.cuda() for t in synth.split_seq(k, P)]
    vs = [t.cuda() for t in synth.split_seq(v, P)]
    rc = rank_chunks(chunks or [H], H, P)
    o_ref, l_ref = relayout_path(qs, ks, vs, P, H, rc, causal)
    o_f, l_f = fused_path(qs, ks, vs, P, H, rc, causal)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    if (S // P) % 128 == 0:  # same tile grid: bitwise
        for a, b in zip(o_f, o_ref):
            assert torch.equal(a, b)
        assert torch.equal(l_f, l_ref)
    else:
        assert_close(torch.cat(o_f, dim=1), torch.cat(o_ref, dim=1), l_f, l_ref)
    ref = oracle.attention(to64(q), to64(k), to64(v), causal=causal)
    assert_close(torch.cat(o_f, dim=1), ref[0], l_f, ref[1])


def test_one_rank_leaves_other_heads_untouched():
    B, S, H, D, P = 1, 1000, 4, 128, 4
    q, k, v = synth.qkv(B, S, H, D, seed=7, scale=0.5)
    qs = [t.cuda() for t in synth.split_seq(q, P)]
    ks = [t.cuda() for t in synth.split_seq(k, P)]
    vs = [t.cuda() for t in synth.split_seq(v, P)]
    o_seq = [torch.full_like(qs[0], 3.0) for _ in range(P)]
    lse = torch.full((B, H, S), 5.0, device="cuda")
    spattn.sp_attn_fwd_seq_sharded(qs, ks, vs, o_seq, lse, heads=(2, 1))
    torch.cuda.synchronize()
    o = torch.cat(o_seq, dim=1)
    ref = oracle.attention(to64(q[:, :, 2:3]), to64(k[:, :, 2:3]), to64(v[:, :, 2:3]))
    assert_close(o[:, :, 2:3], ref[0], lse[:, 2:3], ref[1])
    others = [0, 1, 3]
    assert torch.all(o[:, :, others] == 3.0) and torch.all(lse[:, others] == 5.0)


def test_invalid_arguments_are_rejected():
    B, S, H, D, P = 1, 1000, 4, 128, 4
    qs = [torch.zeros((B, S // P, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    os_ = [torch.zeros_like(qs[0]) for _ in range(P)]
    with pytest.raises(spattn.SpError):  # heads out of range
        spattn.sp_attn_fwd_seq_sharded(qs, qs, qs, os_, heads=(3, 2))
    with pytest.raises(spattn.SpError):  # chunks not summing to the head count
        spattn.sp_attn_fwd_seq_sharded(qs, qs, qs, os_, heads=(0, 4), head_chunks=[1, 2])
    with pytest.raises(spattn.SpError):  # output overlapping an input
        spattn.sp_attn_fwd_seq_sharded(qs, qs, qs, [qs[0]] + os_[1:])
    many = [torch.zeros((1, 128, 1, 64), dtype=torch.bfloat16, device="cuda") for _ in range(9)]
    with pytest.raises(spattn.SpError):  # more shards than SP_MAX_SHARDS
        spattn.sp_attn_fwd_seq_sharded(many, many, many, [torch.zeros_like(t) for t in many])
