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
