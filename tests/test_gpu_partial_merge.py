"""KV blocks merged in place into a running result (sp_attn_fwd_partial_merge) against the fp64 oracle.

A ring's rounds are the first block's partial (sp_attn_fwd_partial) followed by merges of every later block:
the result must equal full attention over all keys (the oracle's unsplit definition) in any block order,
rows that see no key of a block must keep the running result bit for bit, and a running lse of -inf must
keep whatever o_acc holds out of the sum."""
import math

import pytest
import torch

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


def _blocks(S, n, tile_aligned=False):
    blk = -(-S // n)
    if tile_aligned:
        blk = -(-blk // 128) * 128
    return [(i * blk, min(S, (i + 1) * blk)) for i in range(n) if i * blk < S]


def _ring(q, k, v, blocks, causal, mask=None, start="partial"):
    B, S, H, D = q.shape
    o_acc = torch.full((B, S, H, D), float("nan"), device="cuda")
    lse = torch.empty((B, H, S), device="cuda")
    rest = blocks
    if start == "partial":
        a, e = blocks[0]
        spattn.sp_attn_fwd_partial(q, k, v, o_acc, lse, a, e, causal=causal, block_mask=mask)
        rest = blocks[1:]
    else:  # an empty running result: lse = -inf, o_acc anything (NaN here)
        lse.fill_(-math.inf)
    for a, e in rest:
        spattn.sp_attn_fwd_partial_merge(q, k, v, o_acc, lse, a, e, causal=causal, block_mask=mask)
    st, bits = spattn.sp_check_device_error_bits()
    assert st == spattn.SP_OK, hex(bits)
    return o_acc, lse


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("order", ["forward", "reverse", "shuffled"])
def test_ring_of_merges_equals_full_attention(D, causal, order):
    B, S, H = 2, 1500, 3
    q, k, v = synth.qkv(B, S, H, D, seed=D + 3 * causal, scale=0.5)
    ref = oracle.attention(to64(q), to64(k), to64(v), causal=causal)
    blocks = _blocks(S, 5)
    if order == "reverse":
        blocks = blocks[::-1]
    elif order == "shuffled":
        blocks = [blocks[i] for i in (2, 0, 4, 1, 3)]
    o, lse = _ring(q.cuda(), k.cuda(), v.cuda(), blocks, causal)
    assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("causal", [False, True])
def test_merges_from_an_empty_running_result(causal):
    """lse_acc = -inf everywhere and o_acc = NaN: every block is merged, none written first; o_acc's NaN
    never reaches the result."""
    B, S, H, D = 1, 1000, 2, 128
    q, k, v = synth.qkv(B, S, H, D, seed=11, scale=0.5)
    ref = oracle.attention(to64(q), to64(k), to64(v), causal=causal)
    o, lse = _ring(q.cuda(), k.cuda(), v.cuda(), _blocks(S, 3), causal, start="empty")
    assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("D", [64, 128])
def test_rows_without_keys_keep_the_running_result(D):
    """A causal block [640, 1000) merged into an arbitrary running result: rows before 640 see no key and
    stay bit for bit; every other row equals the oracle's merge of the running result with the block's
    partial."""
    B, S, H = 1, 1000, 2
    q, k, v = synth.qkv(B, S, H, D, seed=D, scale=0.5)
    g = torch.Generator().manual_seed(4)
    o0 = torch.randn((B, S, H, D), generator=g)
    l0 = 2.0 * torch.randn((B, H, S), generator=g)
    o_acc, lse = o0.cuda(), l0.cuda()
    spattn.sp_attn_fwd_partial_merge(q.cuda(), k.cuda(), v.cuda(), o_acc, lse, 640, 1000, causal=True)
    assert spattn.sp_check_device_error() == spattn.SP_OK
    oc, lc = o_acc.cpu(), lse.cpu()
    assert torch.equal(oc[:, :640], o0[:, :640]) and torch.equal(lc[:, :, :640], l0[:, :, :640])
    part = oracle.attention(to64(q), to64(k), to64(v), causal=True, kv_begin=640, kv_end=1000)
    ref_o, ref_l = oracle.merge([to64(o0), part[0]], [to64(l0), part[1]])
    assert_close(oc[:, 640:], ref_o[:, 640:], lc[:, :, 640:], ref_l[:, :, 640:])


def test_empty_block_changes_nothing():
    B, S, H, D = 1, 300, 2, 64
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=1))
    o_acc = torch.randn((B, S, H, D), device="cuda")
    lse = torch.randn((B, H, S), device="cuda")
    o0, l0 = o_acc.clone(), lse.clone()
    spattn.sp_attn_fwd_partial_merge(q, k, v, o_acc, lse, 200, 200)
    torch.cuda.synchronize()
    assert torch.equal(o_acc, o0) and torch.equal(lse, l0)


@pytest.mark.parametrize("causal", [False, True])
def test_masked_ring_of_merges(causal):
    """With a block mask (single-CTA kernel, one staging buffer per warp): tile-aligned blocks."""
    B, S, H, D = 1, 1200, 3, 128
    q, k, v = synth.qkv(B, S, H, D, seed=13, scale=0.5)
    mask = synth.block_mask(H, S, seed=13)
    ref = oracle.attention(to64(q), to64(k), to64(v), causal=causal, block_mask=mask.numpy())
    o, lse = _ring(q.cuda(), k.cuda(), v.cuda(), _blocks(S, 4, tile_aligned=True), causal, mask=mask.cuda())
    assert_close(o, ref[0], lse, ref[1])


def test_merging_launches_agree_with_materialised_partials():
    """The in-place merges and the standalone re-merge of materialised partials compute the same
    log-sum-exp rule in fp32: they agree far inside the attention tolerance."""
    B, S, H, D = 1, 2048, 4, 128
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=21, scale=0.5))
    blocks = _blocks(S, 4)
    o, lse = _ring(q, k, v, blocks, True)
    parts_o = [torch.empty((B, S, H, D), device="cuda") for _ in blocks]
    parts_l = [torch.empty((B, H, S), device="cuda") for _ in blocks]
    for (a, e), po, pl in zip(blocks, parts_o, parts_l):
        spattn.sp_attn_fwd_partial(q, k, v, po, pl, a, e, causal=True)
    om = torch.empty((B, S, H, D), device="cuda")
    lm = torch.empty((B, H, S), device="cuda")
    spattn.sp_merge_partials(parts_o, parts_l, om, lm)
    torch.cuda.synchronize()
    assert_close(o, om, lse, lm, o_max_abs=1e-4, o_rel_l2=1e-5, lse_max_abs=1e-5)
