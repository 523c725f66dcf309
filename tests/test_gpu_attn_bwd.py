"""Attention backward on the GPU (sp_attn_bwd: delta, dK/dV and dQ kernels through the C ABI) against the
fp64 oracle's exact gradients.

Tolerance (derived from the arithmetic): p and ds are rounded to bf16 for the tensor cores and the
gradients are written in bf16 (each a relative rounding of at most 2^-9, about 2e-3), o enters delta in
bf16, and sums run over up to S terms in fp32.  Per gradient tensor: ||x - y||_2 / ||y||_2 <= 1e-2 and
max |x - y| <= 2e-2 * max |y|, with the norms floored at 1e-3 (per element): a reference that is exactly zero
(dq and dk with a single key) is compared absolutely."""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import to64
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu
REL_L2 = 1e-2
MAX_REL = 2e-2


def close(x, ref, name):
    x = to64(x)
    d = x - ref
    rel = np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-3 * np.sqrt(ref.size))
    mx = np.max(np.abs(d)) / max(np.max(np.abs(ref)), 1e-3)
    assert np.all(np.isfinite(x)), name
    assert rel <= REL_L2 and mx <= MAX_REL, (name, rel, mx)
    return rel, mx


def run_bwd(q, k, v, do, causal):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    B, S, H, D = q.shape
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd(qd, kd, vd, o, lse, causal=causal)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    spattn.sp_attn_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, causal=causal)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    return dq, dk, dv


@pytest.mark.parametrize("B,S,H,D,causal", [
    (1, 256, 2, 128, False), (1, 256, 2, 128, True), (2, 1000, 3, 128, False), (1, 1000, 3, 128, True),
    (1, 640, 2, 64, False), (2, 383, 2, 64, True), (1, 129, 1, 128, True), (3, 1, 2, 64, False),
])
def test_bwd_matches_oracle(B, S, H, D, causal):
    q, k, v = synth.qkv(B, S, H, D, seed=S + H + D, scale=0.5)
    g = torch.Generator().manual_seed(S + 7)
    do = torch.randn((B, S, H, D), generator=g).to(torch.bfloat16)
    dq, dk, dv = run_bwd(q, k, v, do, causal)
    rq, rk, rv = oracle.attention_bwd(to64(q), to64(k), to64(v), to64(do), causal=causal)
    close(dq, rq, "dq")
    close(dk, rk, "dk")
    close(dv, rv, "dv")


def test_bwd_deterministic():
    B, S, H, D = 1, 700, 2, 128
    q, k, v = synth.qkv(B, S, H, D, seed=3, scale=0.5)
    do = torch.randn((B, S, H, D), generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    a = run_bwd(q, k, v, do, True)
    b = run_bwd(q, k, v, do, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("causal", [False, True])
def test_ring_block_backward_sums_to_full(causal):
    """KV blocks [0,256), [256,512), [512,768), [768,1000) with the merged forward result: each block's dk and
    dv rows equal the full backward's bit for bit (same per-key-tile arithmetic), and the fp32 sum of the
    blocks' dq contributions matches the oracle and the full backward's dq."""
    B, S, H, D = 1, 1000, 2, 128
    q, k, v = synth.qkv(B, S, H, D, seed=41, scale=0.5)
    do = torch.randn((B, S, H, D), generator=torch.Generator().manual_seed(42)).to(torch.bfloat16)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd(qd, kd, vd, o, lse, n_kv_blocks=4, causal=causal)  # KV blocks + merge, as in a ring
    full = [torch.empty_like(qd) for _ in range(3)]
    spattn.sp_attn_bwd(qd, kd, vd, o, dod, lse, *full, causal=causal)
    dq_acc = torch.zeros((B, S, H, D), dtype=torch.float32, device="cuda")
    dk = torch.full_like(qd, float("nan"))
    dv = torch.full_like(qd, float("nan"))
    for a, e in ((0, 256), (256, 512), (512, 768), (768, 1000)):
        spattn.sp_attn_bwd_partial(qd, kd, vd, o, dod, lse, dq_acc, dk, dv, a, e, causal=causal)
    dq = spattn.sp_convert_f32_to_bf16(dq_acc, torch.empty_like(qd))
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    assert torch.equal(dk, full[1]) and torch.equal(dv, full[2])
    rq, rk, rv = oracle.attention_bwd(to64(q), to64(k), to64(v), to64(do), causal=causal)
    close(dq, rq, "dq")
    close(dk, rk, "dk")
    close(dv, rv, "dv")
    close(dq, to64(full[0]), "dq vs full")


def test_partial_backward_rejects_unaligned_block():
    q = torch.zeros((1, 512, 1, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 512), device="cuda")
    acc = torch.zeros((1, 512, 1, 64), device="cuda")
    with pytest.raises(spattn.SpError):
        spattn.sp_attn_bwd_partial(q, q, q, q, q, lse, acc, torch.empty_like(q), torch.empty_like(q), 100, 300)
