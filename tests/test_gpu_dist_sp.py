"""The multi-process sequence-parallel schemes (sequence_head_attention_b200/dist.py) with the library's
kernels and NCCL, on one GPU as a single rank: the collectives are real (a one-rank all-to-all, a ring of
one), the kernels are the ones every rank runs, and the result must be full attention (oracle)."""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import oracle
from tests.helpers import assert_close, to64
from sequence_head_attention_b200 import dist as sp_dist
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


@pytest.fixture
def nccl_one_rank():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


def test_ulysses_and_ring_with_library_kernels(nccl_one_rank):
    B, S, H, D = 1, 2048, 8, 128
    q, k, v = synth.qkv(B, S, H, D, seed=3, scale=0.5)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ref = oracle.attention(to64(q), to64(k), to64(v))
    o1 = torch.empty_like(qd)
    l1 = torch.empty((B, H, S), device="cuda")
    spattn.sp_attn_fwd(qd, kd, vd, o1, l1, head_chunks=[3, 5])
    for stages in (1, 3):
        ul = sp_dist.UlyssesAttention(B, S, H, D, head_chunks=[3, 5], device="cuda", stages=stages)
        o = ul.forward(qd, kd, vd)
        torch.cuda.synchronize()
        assert spattn.sp_check_device_error() == spattn.SP_OK
        assert_close(o, ref[0], ul.lse_heads(), ref[1])
        # same kernels, same tiles (S a multiple of 128), per-head arithmetic independent of the stages
        assert torch.equal(o, o1) and torch.equal(ul.lse_heads(), l1)
    refc = oracle.attention(to64(q), to64(k), to64(v), causal=True)
    ring = sp_dist.RingAttention(B, S, H, D, causal=True, device="cuda")
    o2 = ring.forward(qd, kd, vd)
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK
    assert ring.rounds == [(0, 0, "causal")]
    assert_close(o2, refc[0], ring.lse, refc[1])
