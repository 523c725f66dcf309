"""The allocation-free block-sparse entry point, for callers that cannot allocate device memory (a
serving path that must not block on an allocation's device synchronisation, a plug-in whose host
framework owns every allocation, a real-time loop with no allocation after start-up).

It must give what the workspace-based entry point gives, call after call, although every call reuses
the same fixed scratch array inside the library.  This file is collected last on purpose, and passes
both on its own in a fresh process and after the rest of the suite.
"""
import pytest
import torch

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


def _with_workspace(q, k, v, mask, causal):
    B, S, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd(q, k, v, o, lse, causal=causal, block_mask=mask)
    return o, lse


def _no_alloc(q, k, v, mask, causal):
    B, S, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd_sparse_noalloc(q, k, v, o, lse, mask, causal=causal)
    return o, lse


@pytest.mark.parametrize("first,second", [
    ((1, 4096, 8, 128, False, 1), (1, 2048, 16, 128, True, 2)),
    ((2, 1000, 3, 64, True, 3), (1, 32768, 40, 128, False, 0)),   # second call: the full block-sparse shape
])
def test_no_alloc_matches_workspace_entry_point_two_calls_in_a_row(first, second):
    """Two calls in a row (the second reuses the scratch the first left behind): each equals the
    workspace-based entry point bit for bit, since both run the same kernels on the same tile list, and
    sampled rows of each match the fp64 oracle within the attention tolerance."""
    for B, S, H, D, causal, seed in (first, second):
        q, k, v = synth.qkv(B, S, H, D, seed=seed, scale=0.5)
        mask = synth.block_mask(H, S, seed=seed)
        qd, kd, vd, md = q.cuda(), k.cuda(), v.cuda(), mask.cuda()
        ref_o, ref_l = _with_workspace(qd, kd, vd, md, causal)
        o, lse = _no_alloc(qd, kd, vd, md, causal)
        st, bits = spattn.sp_check_device_error_bits()
        assert st == spattn.SP_OK, hex(bits)
        assert torch.equal(o, ref_o) and torch.equal(lse, ref_l)
        rows = synth.sample_rows(S, 24, seed=seed, must=[0, S - 1])
        ref = oracle.attention(to64(q), to64(k), to64(v), causal=causal, block_mask=mask.numpy(), rows=rows)
        r = torch.tensor(rows, device="cuda")
        assert_close(o[:, r], ref[0], lse[:, :, r], ref[1])


def test_no_alloc_refuses_masks_beyond_its_scratch():
    # H * ceil(S/128) = 20000 tile rows > SP_NOALLOC_MAX_TILE_ROWS (16384): refused before any launch
    L = spattn.lib()
    st = L.sp_attn_fwd_sparse_noalloc(16, 16, 16, 16, None, 1, 128 * 500, 40, 128, 0, 16, None)
    assert st == spattn.SP_ERR_UNSUPPORTED
    # H * ceil(S/128)^2 = 4 * 1024^2 > SP_NOALLOC_MAX_TILES
    st = L.sp_attn_fwd_sparse_noalloc(16, 16, 16, 16, None, 1, 128 * 1024, 4, 128, 0, 16, None)
    assert st == spattn.SP_ERR_UNSUPPORTED
    st = L.sp_attn_fwd_sparse_noalloc(16, 16, 16, 16, None, 1, 1024, 4, 128, 0, None, None)
    assert st == spattn.SP_ERR_INVALID_ARG  # the mask is required
