"""Re-merge of KV-block partials on the GPU against the oracle's log-sum-exp rule."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import spattn

pytestmark = pytest.mark.gpu


def _partials(n, B, S, H, D, seed, empty_before=None):
    """Synthetic partials: o_b ~ N(0,1), lse_b ~ 3 N(0,1); with empty_before[b] = s0, rows s < s0 of block
    b are empty (o = 0, lse = -inf), the structure causal ring partials have."""
    g = torch.Generator().manual_seed(seed)
    os_, ls_ = [], []
    for b in range(n):
        o = torch.randn((B, S, H, D), generator=g)
        l = 3.0 * torch.randn((B, H, S), generator=g)
        if empty_before is not None:
            s0 = empty_before[b]
            o[:, :s0] = 0
            l[:, :, :s0] = -math.inf
        os_.append(o)
        ls_.append(l)
    return os_, ls_


@pytest.mark.parametrize("n,B,S,H,D", [(2, 1, 256, 4, 64), (3, 2, 100, 3, 128), (8, 1, 1000, 5, 128),
                                       (1, 1, 64, 2, 64), (17, 1, 40, 2, 128)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_merge_matches_oracle(n, B, S, H, D, out_dtype):
    empty = [min(S, (S // n) * b) for b in range(n)]
    os_, ls_ = _partials(n, B, S, H, D, seed=n * 7 + S, empty_before=empty)
    ls_[0][:, :, : S // 4] = -math.inf  # some rows with no visible key at all
    os_[0][:, : S // 4] = 0
    ref_o, ref_l = oracle.merge([to64(x) for x in os_], [to64(x) for x in ls_])
    o = torch.empty((B, S, H, D), dtype=out_dtype, device="cuda")
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    spattn.sp_merge_partials([x.cuda() for x in os_], [x.cuda() for x in ls_], o, lse)
    if out_dtype == torch.float32:
        assert_close(o, ref_o, lse, ref_l, o_max_abs=1e-5, o_rel_l2=1e-6, lse_max_abs=1e-5)
    else:
        assert_close(o, ref_o, lse, ref_l)
    # rows where every partial is empty: exactly 0 and -inf
    s_empty = min(S // 4, S // n) if n > 1 else S // 4
    assert torch.all(o[:, :s_empty].float() == 0)
    assert torch.all(torch.isneginf(lse[:, :, :s_empty]))


def test_merge_in_place_and_identities():
    B, S, H, D = 1, 300, 2, 128
    os_, ls_ = _partials(3, B, S, H, D, seed=5)
    ref_o, ref_l = oracle.merge([to64(x) for x in os_], [to64(x) for x in ls_])
    d_o = [x.cuda() for x in os_]
    d_l = [x.cuda() for x in ls_]
    spattn.sp_merge_partials(d_o, d_l, d_o[0], d_l[0])  # in place into part 0
    assert_close(d_o[0], ref_o, d_l[0], ref_l, o_max_abs=1e-5, o_rel_l2=1e-6, lse_max_abs=1e-5)
    # n = 1 is the identity; merging a partial with itself gives lse + ln 2
    o1 = torch.empty_like(d_o[1])
    l1 = torch.empty_like(d_l[1])
    spattn.sp_merge_partials([d_o[1]], [d_l[1]], o1, l1)
    assert torch.equal(o1, d_o[1]) and torch.allclose(l1, d_l[1], atol=1e-6, rtol=0)
    spattn.sp_merge_partials([d_o[1], d_o[1]], [d_l[1], d_l[1]], o1, l1)
    assert torch.allclose(o1, d_o[1], atol=1e-5, rtol=0)
    assert torch.allclose(l1, d_l[1] + math.log(2), atol=1e-5, rtol=0)


def test_merge_full_size_ring_partials_sampled():
    """Eight fp32 partials of the long ring shape [1, 57344, 40, 128], drawn on the GPU from a seeded
    generator with the causal block structure (rows before a block's start are empty); checked on
    sampled rows against the oracle."""
    n, B, S, H, D = 8, 1, 57344, 40, 128
    g = torch.Generator(device="cuda").manual_seed(11)
    blk = S // n
    os_, ls_ = [], []
    for b in range(n):
        o = torch.randn((B, S, H, D), generator=g, device="cuda")
        l = 3.0 * torch.randn((B, H, S), generator=g, device="cuda")
        o[:, : b * blk] = 0
        l[:, :, : b * blk] = -math.inf
        os_.append(o)
        ls_.append(l)
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    spattn.sp_merge_partials(os_, ls_, out, lse)
    rows = torch.tensor(sorted({0, 1, blk - 1, blk, 3 * blk + 5, S - 1} | set(range(7, S, 997))), device="cuda")
    ref_o, ref_l = oracle.merge([to64(x[:, rows]) for x in os_], [to64(x[:, :, rows]) for x in ls_])
    assert_close(out[:, rows], ref_o, lse[:, :, rows], ref_l)
    del os_, ls_
    torch.cuda.empty_cache()
