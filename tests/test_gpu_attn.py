"""Attention on the GPU (tcgen05 kernel through the C ABI) against the fp64 oracle.

Sizes here span several 128-row tiles and ragged tails, so the oracle finishes in seconds and every
output element is compared; the full-size workloads are in test_gpu_full_size.py.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import assert_close, metrics, to64
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


def gpu_attn(q, k, v, chunks=None, n_kv=1, causal=False, mask=None):
    B, S, H, D = q.shape
    o = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    spattn.sp_attn_fwd(q.cuda(), k.cuda(), v.cuda(), o, lse, head_chunks=chunks, n_kv_blocks=n_kv,
                       causal=causal, block_mask=None if mask is None else mask.cuda())
    assert spattn.sp_check_device_error() == spattn.SP_OK
    return o, lse


def ref_attn(q, k, v, causal=False, mask=None, kv_begin=0, kv_end=None):
    return oracle.attention(to64(q), to64(k), to64(v), causal=causal,
                            block_mask=None if mask is None else mask.numpy(), kv_begin=kv_begin,
                            kv_end=kv_end)


def test_tiny_dense_workload():
    """B1 H4 S256 D64, fp32 N(0,1) rounded to bf16, head chunks [1, 3], 2 KV blocks of 128."""
    w = synth.WORKLOADS["tiny_dense"]
    q, k, v, raw = synth.qkv(w.B, w.S, w.H, w.D, seed=0, fp32_source=True)
    ref = ref_attn(q, k, v)
    for n_kv in (1, 2):
        o, lse = gpu_attn(q, k, v, chunks=list(w.head_chunks), n_kv=n_kv)
        assert_close(o, ref[0], lse, ref[1])
    # For information: deviation from attention on the unrounded fp32 inputs.
    ref32 = oracle.attention(*(r.double().numpy() for r in raw))
    m = metrics(o, ref32[0], lse, ref32[1])
    print("tiny_dense vs unrounded fp32 inputs:", m)


def test_megatron_workload_and_rank_order():
    """B4 S128 H32 D128, chunks [8,8,8,8]: output viewed [4, 128, 4096] equals full attention, every
    chunking gives bitwise the same result, and a wrongly ordered concatenation does not match."""
    w = synth.WORKLOADS["megatron"]
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=0)
    ref = ref_attn(q, k, v)
    o, lse = gpu_attn(q, k, v, chunks=list(w.head_chunks))
    assert_close(o, ref[0], lse, ref[1])
    assert tuple(o.view(w.B, w.S, w.H * w.D).shape) == (4, 128, 4096)
    for chunks in (None, [32], [1] * 32, [5, 11, 16]):
        o2, lse2 = gpu_attn(q, k, v, chunks=chunks)
        assert torch.equal(o2, o) and torch.equal(lse2, lse)
    # per-rank 8-head runs, concatenated in rank order == full; rotated order != full
    per = []
    for r in range(4):
        hs = slice(8 * r, 8 * r + 8)
        o_r, _ = gpu_attn(q[:, :, hs].contiguous(), k[:, :, hs].contiguous(), v[:, :, hs].contiguous())
        per.append(o_r.view(w.B, w.S, 8 * w.D))
    cat = torch.cat(per, dim=-1)
    assert torch.equal(cat, o.view(w.B, w.S, -1))
    wrong = torch.cat(per[1:] + per[:1], dim=-1)
    assert metrics(wrong, ref[0].reshape(w.B, w.S, -1))["max_abs"] > 0.5


@pytest.mark.parametrize("B,S,H,D,causal", [
    (2, 1000, 3, 128, False), (2, 1000, 3, 128, True), (1, 1000, 3, 64, False), (1, 1000, 3, 64, True),
    (1, 129, 2, 128, True), (3, 1, 2, 64, False), (1, 383, 2, 128, False), (1, 256, 1, 128, True),
    (1, 640, 2, 128, False),
])
def test_dense_ragged(B, S, H, D, causal):
    q, k, v = synth.qkv(B, S, H, D, seed=S + H, scale=1.0)
    ref = ref_attn(q, k, v, causal=causal)
    o, lse = gpu_attn(q, k, v, causal=causal)
    assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("kv", [(100, 700), (0, 1000), (640, 1000), (128, 256), (999, 1000), (500, 500)])
@pytest.mark.parametrize("causal", [False, True])
def test_partial_block(kv, causal):
    B, S, H, D = 1, 1000, 3, 128
    q, k, v = synth.qkv(B, S, H, D, seed=3, scale=0.5)
    ref = ref_attn(q, k, v, causal=causal, kv_begin=kv[0], kv_end=kv[1])
    o = torch.full((B, S, H, D), float("nan"), device="cuda")
    lse = torch.full((B, H, S), float("nan"), device="cuda")
    spattn.sp_attn_fwd_partial(q.cuda(), k.cuda(), v.cuda(), o, lse, kv[0], kv[1], causal=causal)
    assert spattn.sp_check_device_error() == spattn.SP_OK
    assert_close(o, ref[0], lse, ref[1])
    empty = np.isneginf(ref[1])  # rows that see no key: exactly zero output
    if empty.any():
        oe = o.cpu().numpy().transpose(0, 2, 1, 3)[empty]
        assert np.all(oe == 0)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("kv", [(1100, 1500), (512, 1024), (1400, 1401)])
def test_causal_partial_rows_before_block(D, kv):
    """A causal block over keys [kv_begin, kv_end): query rows before kv_begin see no key.  Whole work
    units of them are not run but filled (O = 0, lse = -inf), batch by batch; every other row matches."""
    B, S, H = 2, 1500, 3
    q, k, v = synth.qkv(B, S, H, D, seed=kv[0] + D, scale=0.5)
    ref = ref_attn(q, k, v, causal=True, kv_begin=kv[0], kv_end=kv[1])
    o = torch.full((B, S, H, D), float("nan"), device="cuda")
    lse = torch.full((B, H, S), float("nan"), device="cuda")
    spattn.sp_attn_fwd_partial(q.cuda(), k.cuda(), v.cuda(), o, lse, kv[0], kv[1], causal=True)
    assert spattn.sp_check_device_error() == spattn.SP_OK
    assert_close(o, ref[0], lse, ref[1])
    oc, lc = o.cpu().numpy(), lse.cpu().numpy()
    assert np.all(oc[:, :kv[0]] == 0) and np.all(np.isneginf(lc[:, :, :kv[0]]))


@pytest.mark.parametrize("n_kv", [2, 3, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_kv_blocks_merge_equals_unsplit(n_kv, causal):
    B, S, H, D = 1, 1000, 2, 128
    q, k, v = synth.qkv(B, S, H, D, seed=n_kv, scale=0.5)
    ref = ref_attn(q, k, v, causal=causal)
    o, lse = gpu_attn(q, k, v, n_kv=n_kv, causal=causal)
    assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("D", [64, 128])
def test_causal_kv_blocks_with_chunks_and_skipped_units(D):
    """n_kv_blocks > 1, causal, uneven head chunks and two batches at a size where the later blocks skip
    whole leading query units (filled 0 / -inf) before the merge: equals the unsplit oracle."""
    B, S, H = 2, 2100, 3
    q, k, v = synth.qkv(B, S, H, D, seed=D + 5, scale=0.5)
    ref = ref_attn(q, k, v, causal=True)
    for n_kv in (2, 3):
        o, lse = gpu_attn(q, k, v, chunks=[1, 2], n_kv=n_kv, causal=True)
        assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_kv", [1, 2])
def test_block_sparse(causal, n_kv):
    B, S, H, D = 1, 1000, 3, 128
    q, k, v = synth.qkv(B, S, H, D, seed=9, scale=0.5)
    mask = synth.block_mask(H, S, seed=9)
    ref = ref_attn(q, k, v, causal=causal, mask=mask)
    o, lse = gpu_attn(q, k, v, causal=causal, mask=mask, n_kv=n_kv)
    assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("causal", [False, True])
def test_block_sparse_kv_blocks_rounded_past_s(causal):
    """With a mask the KV block size is rounded up to whole tiles: S = 1200 in 7 blocks gives blocks of
    256 keys, so blocks 5 and 6 would start at or past S.  They hold no key and are dropped; the keys of
    the last tile (1152..1199) are counted once, and the result equals the unsplit oracle."""
    B, S, H, D = 1, 1200, 3, 128
    q, k, v = synth.qkv(B, S, H, D, seed=12, scale=0.5)
    mask = synth.block_mask(H, S, seed=12)
    ref = ref_attn(q, k, v, causal=causal, mask=mask)
    for n_kv in (7, 10):
        o, lse = gpu_attn(q, k, v, causal=causal, mask=mask, n_kv=n_kv)
        assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("kind", ["diagonal", "random", "first_and_diagonal"])
def test_block_sparse_lanes_split_keys(D, causal, kind):
    """Masked launches put both lanes on one query tile, dealing its kept key tiles to them in turn: rows
    with one kept tile (the second lane gets none), an odd or even count, an odd number of query tiles
    (S = 1100: the last pair has one tile) and two batches, all against the oracle."""
    B, S, H = 2, 1100, 3
    T = (S + 127) // 128
    q, k, v = synth.qkv(B, S, H, D, seed=D + causal, scale=0.5)
    if kind == "diagonal":
        mask = torch.zeros((H, T, T), dtype=torch.uint8)
        mask[:, torch.arange(T), torch.arange(T)] = 1
    elif kind == "first_and_diagonal":
        mask = torch.zeros((H, T, T), dtype=torch.uint8)
        mask[:, torch.arange(T), torch.arange(T)] = 1
        mask[:, :, 0] = 1
    else:
        mask = synth.block_mask(H, S, seed=D)
    ref = ref_attn(q, k, v, causal=causal, mask=mask)
    o, lse = gpu_attn(q, k, v, causal=causal, mask=mask)
    assert_close(o, ref[0], lse, ref[1])


def test_block_sparse_partial_and_empty_rows():
    B, S, H, D = 1, 1000, 3, 64
    q, k, v = synth.qkv(B, S, H, D, seed=4, scale=0.5)
    mask = synth.block_mask(H, S, seed=4)
    mask[0, :, :] = 0  # head 0 keeps nothing: every row empty
    for kv in ((256, 1000), (0, 384)):
        ref = ref_attn(q, k, v, mask=mask, kv_begin=kv[0], kv_end=kv[1])
        o = torch.empty((B, S, H, D), device="cuda")
        lse = torch.empty((B, H, S), device="cuda")
        spattn.sp_attn_fwd_partial(q.cuda(), k.cuda(), v.cuda(), o, lse, kv[0], kv[1], block_mask=mask.cuda())
        assert spattn.sp_check_device_error() == spattn.SP_OK
        assert_close(o, ref[0], lse, ref[1])
        assert torch.all(o[:, :, 0] == 0) and torch.all(torch.isneginf(lse[:, 0]))


@pytest.mark.parametrize("D", [64, 128])
def test_all_ones_mask_equals_dense(D):
    """A mask that keeps every tile gives the dense result.  Masked launches split each query tile's key
    tiles between the two lanes and merge their partial softmaxes, so the two agree to rounding (the bf16
    outputs may differ by an ulp), and both match the oracle."""
    B, S, H = 1, 700, 2
    q, k, v = synth.qkv(B, S, H, D, seed=21)
    T = (S + 127) // 128
    ref = ref_attn(q, k, v)
    o1, l1 = gpu_attn(q, k, v, mask=torch.ones((H, T, T), dtype=torch.uint8))
    o2, l2 = gpu_attn(q, k, v)
    assert_close(o1, ref[0], l1, ref[1])
    assert_close(o1, o2, l1, l2, lse_max_abs=1e-5)


def test_large_scores_stay_finite():
    B, S, H, D = 1, 512, 2, 128
    q, k, v = synth.qkv(B, S, H, D, seed=5)
    q = (q.float() * 8).to(torch.bfloat16)
    ref = ref_attn(q, k, v, causal=True)
    o, lse = gpu_attn(q, k, v, causal=True)
    assert_close(o, ref[0], lse, ref[1])


def test_deterministic_and_outputs_confined():
    B, S, H, D = 1, 900, 2, 128
    q, k, v = synth.qkv(B, S, H, D, seed=8)
    n = B * S * H * D
    guard = 1 << 14
    buf = torch.full((n + 2 * guard,), 7777, dtype=torch.int16, device="cuda")
    o = buf[guard:guard + n].view(torch.bfloat16).view(B, S, H, D)
    lse = torch.empty((B, H, S), device="cuda")
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    spattn.sp_attn_fwd(qd, kd, vd, o, lse, causal=True)
    first = o.clone()
    spattn.sp_attn_fwd(qd, kd, vd, o, lse, causal=True)
    assert torch.equal(first, o)
    assert torch.all(buf[:guard] == 7777) and torch.all(buf[-guard:] == 7777)


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier that nothing completes gives up after its limit and reports SP_ERR_TIMEOUT;
    the context stays usable."""
    spattn.sp_debug_wait_timeout(2_000_000)  # 2 ms
    assert spattn.sp_check_device_error() == spattn.SP_ERR_TIMEOUT
    assert spattn.sp_check_device_error() == spattn.SP_OK  # cleared
    q, k, v = synth.qkv(1, 256, 1, 64, seed=1)
    ref = ref_attn(q, k, v)
    o, lse = gpu_attn(q, k, v)
    assert_close(o, ref[0], lse, ref[1])


@pytest.mark.parametrize("causal,kv,mask_heads_empty", [(True, (2048, 4096), False), (False, (0, 4096), True),
                                                        (True, (0, 1024), False)])
def test_many_items_per_cta_with_empty_lanes(causal, kv, mask_heads_empty):
    """40 heads x 16 query-tile pairs = 640 work items over at most 148 CTAs, several per CTA, with
    items whose lanes see no key at all (queries before a causal KV block, or heads whose mask keeps
    nothing), mixed with full items; sampled rows against the oracle."""
    B, S, H, D = 1, 4096, 40, 128
    q, k, v = synth.qkv(B, S, H, D, seed=17, scale=0.5)
    mask = None
    if mask_heads_empty:
        mask = synth.block_mask(H, S, seed=17)
        mask[::3] = 0
    rows = synth.sample_rows(S, 48, seed=3, must=[kv[0] - 1, kv[0], 2047, 2048, 4095])
    ref = oracle.attention(to64(q), to64(k), to64(v), causal=causal, rows=rows, kv_begin=kv[0], kv_end=kv[1],
                           block_mask=None if mask is None else mask.numpy())
    o = torch.empty((B, S, H, D), device="cuda")
    lse = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd_partial(q.cuda(), k.cuda(), v.cuda(), o, lse, kv[0], kv[1], causal=causal,
                               block_mask=None if mask is None else mask.cuda())
    st, bits = spattn.sp_check_device_error_bits()
    assert st == spattn.SP_OK, hex(bits)
    r = torch.tensor(rows, device="cuda")
    assert_close(o[:, r], ref[0], lse[:, :, r], ref[1])


def test_concurrent_launches_on_two_streams():
    """Two launches in flight at once on different streams draw different work counters; each result
    equals the same launch run alone, and repeated launches (counters reused after their reset) agree."""
    B, S, H, D = 1, 4096, 8, 128
    qa, ka, va = (t.cuda() for t in synth.qkv(B, S, H, D, seed=31, scale=0.5))
    qb, kb, vb = (t.cuda() for t in synth.qkv(B, S, H, D, seed=32, scale=0.5))
    ref_a, ref_b = gpu_attn(qa, ka, va, causal=True), gpu_attn(qb, kb, vb)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = []
    for _ in range(70):  # more launches than there are counter slots
        oa = torch.empty_like(ref_a[0]); la = torch.empty_like(ref_a[1])
        ob = torch.empty_like(ref_b[0]); lb = torch.empty_like(ref_b[1])
        spattn.sp_attn_fwd(qa, ka, va, oa, la, causal=True, stream=s1)
        spattn.sp_attn_fwd(qb, kb, vb, ob, lb, stream=s2)
        outs.append((oa, la, ob, lb))
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    for oa, la, ob, lb in outs:
        assert torch.equal(oa, ref_a[0]) and torch.equal(la, ref_a[1])
        assert torch.equal(ob, ref_b[0]) and torch.equal(lb, ref_b[1])


def test_binding_refuses_host_or_undersized_masks():
    """Masks the kernels would read out of bounds (a host tensor, too few tiles) and a wrong lse are
    refused by the binding before the library is called."""
    B, S, H, D = 1, 1000, 3, 128
    q, k, v = (t.cuda() for t in synth.qkv(B, S, H, D, seed=2))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), device="cuda")
    good = synth.block_mask(H, S, seed=2)
    bad = [good, good[:, :4, :4].contiguous().cuda(), good[:2].contiguous().cuda()]
    items = torch.zeros(1, dtype=torch.int32, device="cuda")
    for m in bad:
        with pytest.raises(ValueError):
            spattn.sp_attn_fwd(q, k, v, o, lse, block_mask=m)
        with pytest.raises(ValueError):
            spattn.sp_attn_fwd_sparse_noalloc(q, k, v, o, lse, m)
        with pytest.raises(ValueError):
            spattn.sp_attn_fwd_items(q, k, v, o, lse, items, block_mask=m)
        with pytest.raises(ValueError):
            spattn.sp_attn_fwd_partial(q, k, v, o.float(), lse, 0, S, block_mask=m)
    with pytest.raises(ValueError):
        spattn.sp_attn_fwd_sparse_noalloc(q, k, v, o, lse[:, :, :-1], good.cuda())
    with pytest.raises(ValueError):
        spattn.sp_attn_fwd_sparse_noalloc(q, k, v, o, lse.cpu(), good.cuda())
