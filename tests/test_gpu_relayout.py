"""Ulysses seq<->head relayout on the GPU: bit-exact against the oracle's index formula."""
import numpy as np
import pytest
import torch

import oracle
from sequence_head_attention_b200 import spattn, synth

pytestmark = pytest.mark.gpu


def _bits(t):
    """View any tensor's bytes as int16/uint8 numpy for exact comparison."""
    t = t.detach().cpu().contiguous()
    if t.element_size() == 2:
        return t.view(torch.int16).numpy()
    if t.element_size() == 4:
        return t.view(torch.int32).numpy()
    if t.element_size() == 8:
        return t.view(torch.int64).numpy()
    return t.view(torch.uint8).numpy()


@pytest.mark.parametrize("P,B,S,H,D,dtype", [
    (4, 1, 32760, 40, 128, torch.bfloat16),   # video-DiT shape, 4 simulated ranks
    (4, 2, 1000, 8, 64, torch.bfloat16),
    (2, 1, 6, 2, 8, torch.float32),
    (1, 1, 256, 4, 64, torch.bfloat16),       # P = 1 is the identity
    (8, 1, 64, 8, 16, torch.uint8),
    (3, 2, 9, 6, 2, torch.float64),
])
def test_seq_to_head_and_back_bit_exact(P, B, S, H, D, dtype):
    g = torch.Generator().manual_seed(P * 1000 + S)
    if dtype == torch.uint8:
        full = torch.randint(0, 256, (B, S, H, D), generator=g, dtype=torch.uint8)
    else:
        full = torch.randn((B, S, H, D), generator=g, dtype=torch.float32).to(dtype)
    shards = synth.split_seq(full, P)
    dev_in = [s.cuda() for s in shards]
    dev_out = [torch.empty((B, S, H // P, D), dtype=dtype, device="cuda") for _ in range(P)]
    spattn.sp_seq_to_head_relayout(dev_in, dev_out)
    ref = oracle.seq_to_head([_bits(s) for s in shards], H)
    for r in range(P):
        assert np.array_equal(_bits(dev_out[r]), ref[r]), f"rank {r}"
    back = [torch.empty_like(s) for s in dev_in]
    spattn.sp_head_to_seq_relayout(dev_out, back)
    ref_back = oracle.head_to_seq(ref, S)
    for r in range(P):
        assert np.array_equal(_bits(back[r]), ref_back[r])
        assert np.array_equal(_bits(back[r]), _bits(shards[r]))  # round trip is the identity
    torch.cuda.synchronize()
    assert spattn.sp_check_device_error() == spattn.SP_OK


def test_relayout_leaves_bytes_outside_outputs_untouched():
    P, B, S, H, D = 2, 1, 64, 4, 64
    x = torch.randn((B, S, H, D)).to(torch.bfloat16)
    ins = [s.cuda() for s in synth.split_seq(x, P)]
    guard = 4096
    outs, bufs = [], []
    for _ in range(P):
        n = B * S * (H // P) * D
        buf = torch.full((n + 2 * guard,), 12345, dtype=torch.int16, device="cuda")
        bufs.append(buf)
        outs.append(buf[guard:guard + n].view(torch.bfloat16).view(B, S, H // P, D))
    spattn.sp_seq_to_head_relayout(ins, outs)
    for buf in bufs:
        assert torch.all(buf[:guard] == 12345) and torch.all(buf[-guard:] == 12345)


@pytest.mark.parametrize("P,B,S,H,D,dtype", [
    (4, 1, 8190, 40, 128, torch.bfloat16),    # one video-DiT rank's sequence shard, 4 ranks
    (8, 2, 300, 8, 64, torch.bfloat16),
    (2, 1, 7, 6, 8, torch.float32),
    (1, 1, 100, 4, 64, torch.bfloat16),       # P = 1: a copy
    (3, 2, 5, 9, 2, torch.float64),
])
def test_split_and_merge_heads_bit_exact(P, B, S, H, D, dtype):
    """The local halves of a multi-process exchange: every head group equals the oracle's, bytes exact,
    and merging them back gives the shard; nothing outside the outputs is written."""
    g = torch.Generator().manual_seed(P * 100 + S)
    x = torch.randn((B, S, H, D), generator=g, dtype=torch.float32).to(dtype)
    ref = oracle.split_heads(_bits(x), P)
    xd = x.cuda()
    guard = 1 << 12
    outs_buf = [torch.full((B * S * (H // P) * D + 2 * guard,), 7, dtype=dtype, device="cuda") for _ in range(P)]
    outs = [b[guard:-guard].view(B, S, H // P, D) for b in outs_buf]
    spattn.sp_split_heads(xd, outs)
    back = torch.empty_like(xd)
    spattn.sp_merge_heads(outs, back)
    torch.cuda.synchronize()
    for r in range(P):
        assert np.array_equal(_bits(outs[r]), ref[r])
        assert torch.all(outs_buf[r][:guard] == 7) and torch.all(outs_buf[r][-guard:] == 7)
    assert np.array_equal(_bits(back), oracle.merge_heads(ref))
    assert np.array_equal(_bits(back), _bits(x))
    # stages of a chunked exchange: heads [h0, h0 + n) of every group, against the oracle's groups sliced
    Hl = H // P
    cuts = [0, (Hl + 1) // 2, Hl] if Hl > 1 else [0, 1]
    back2 = torch.zeros_like(xd)
    for h0, h1 in zip(cuts[:-1], cuts[1:]):
        part = [torch.empty((B, S, h1 - h0, D), dtype=dtype, device="cuda") for _ in range(P)]
        spattn.sp_split_heads(xd, part, heads=(h0, h1 - h0))
        spattn.sp_merge_heads(part, back2, heads=(h0, h1 - h0))
        torch.cuda.synchronize()
        for r in range(P):
            assert np.array_equal(_bits(part[r]), ref[r][:, :, h0:h1])
    assert np.array_equal(_bits(back2), _bits(x))
