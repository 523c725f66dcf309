"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle-side checks.

This module holds no attention arithmetic: it only draws random numbers on the CPU and rounds them to
the storage type.  Both the CUDA path and the oracle receive exactly these values.

Workloads (sizes from the pages' sequence lengths, head counts and head dims; no public data set or
trained model is used, these stand in for the video-generation sequences of 31K-56K tokens, the DiT
block-sparse masks and the tensor-parallel demo):

=====================  ====================================================================================
``tiny_dense``         B1 S256 H4 D64, fp32 N(0,1) rounded to bf16, non-causal, head chunks [1, 3],
                       2 KV blocks of 128.
``megatron``           B4 S128 H32 D128 (hidden 4096), N(0,1), non-causal, head chunks [8, 8, 8, 8]
                       ("LLM Lab Notes 05", section 2: batch 4, seq 128, hidden 4096, 32 heads).
``video_dit``          B1 S32760 H40 D128, N(0,1)*0.5, non-causal, head chunks [3, 7, 10, 10, 10],
                       P=4 ranks for the seq<->head relayout ("HCMS", abstract: 31K-56K tokens).
``ring_causal``        B1 S57344 H40 D128, N(0,1)*0.5, causal, 8 KV blocks of 7168 re-merged.
``block_sparse``       B1 S32768 H40 D128, N(0,1)*0.5, non-causal, per-head 128x128 tile mask with
                       density ~ U[0.1, 0.9] per head, tiles i.i.d. Bernoulli, diagonal kept.
=====================  ====================================================================================
"""
from __future__ import annotations

import dataclasses

import torch

TILE = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int
    H: int
    D: int
    scale: float = 1.0
    causal: bool = False
    head_chunks: tuple = ()
    n_kv_blocks: int = 1
    ranks: int = 1
    sparse: bool = False
    fp32_source: bool = False

    @property
    def n_tiles(self) -> int:
        return (self.S + TILE - 1) // TILE

    def flops(self, density: float = 1.0) -> float:
        """4 * B * H * S^2 * D * density, halved when causal (the metric's algorithmic count)."""
        f = 4.0 * self.B * self.H * self.S * self.S * self.D * density
        return f / 2.0 if self.causal else f


WORKLOADS = {
    "tiny_dense": Workload("tiny_dense", 1, 256, 4, 64, 1.0, False, (1, 3), 2, 1, False, True),
    "megatron": Workload("megatron", 4, 128, 32, 128, 1.0, False, (8, 8, 8, 8), 1, 4),
    "video_dit": Workload("video_dit", 1, 32760, 40, 128, 0.5, False, (3, 7, 10, 10, 10), 1, 4),
    "ring_causal": Workload("ring_causal", 1, 57344, 40, 128, 0.5, True, (40,), 8, 1),
    "block_sparse": Workload("block_sparse", 1, 32768, 40, 128, 0.5, False, (40,), 1, 1, True),
}


def qkv(B: int, S: int, H: int, D: int, seed: int = 0, scale: float = 1.0, fp32_source: bool = False):
    """Q, K, V as bf16 CPU tensors [B, S, H, D], drawn in that order from one seeded CPU generator.

    Values are N(0, 1) * scale in fp32, rounded to bf16 (round to nearest even).  ``fp32_source`` also
    returns the fp32 draws before rounding (for reporting the deviation against unrounded inputs).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    out, raw = [], []
    for _ in range(3):
        t = torch.randn((B, S, H, D), generator=g, dtype=torch.float32)
        if scale != 1.0:
            t.mul_(scale)
        raw.append(t if fp32_source else None)
        out.append(t.to(torch.bfloat16))
    if fp32_source:
        return out[0], out[1], out[2], raw
    return out[0], out[1], out[2]


def block_mask(H: int, S: int, seed: int = 0, lo: float = 0.1, hi: float = 0.9, tile: int = TILE):
    """Per-head tile mask uint8 [H, T, T], T = ceil(S / tile).

    Head h draws its density p_h ~ U[lo, hi]; every off-diagonal tile is kept with probability p_h,
    independently; diagonal tiles are always kept.  Uses its own generator seeded with 1000 + seed.
    """
    T = (S + tile - 1) // tile
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + int(seed))
    p = lo + (hi - lo) * torch.rand((H, 1, 1), generator=g, dtype=torch.float64)
    u = torch.rand((H, T, T), generator=g, dtype=torch.float64)
    m = (u < p).to(torch.uint8)
    idx = torch.arange(T)
    m[:, idx, idx] = 1
    return m


def split_seq(x: torch.Tensor, P: int):
    """Split a [B, S, H, D] tensor into P contiguous sequence shards [B, S/P, H, D] (separate copies)."""
    B, S, H, D = x.shape
    assert S % P == 0
    return [x[:, r * (S // P):(r + 1) * (S // P)].contiguous() for r in range(P)]


def sample_rows(S: int, n: int, seed: int = 0, must=()):
    """Stratified sample of query positions: the given ``must`` rows, rows 0 and S-1, the whole of the
    last (possibly ragged) tile's first and last rows, then one random row per stratum of S/n."""
    g = torch.Generator(device="cpu")
    g.manual_seed(7919 + int(seed))
    last_tile = ((S - 1) // TILE) * TILE
    rows = {0, S - 1, last_tile, min(S - 1, last_tile + 1)}
    rows.update(int(r) for r in must if 0 <= int(r) < S)
    n_rand = max(0, n - len(rows))
    if n_rand:
        edges = torch.linspace(0, S, n_rand + 1).long()
        for a, b in zip(edges[:-1].tolist(), edges[1:].tolist()):
            if b > a:
                rows.add(a + int(torch.randint(0, b - a, (1,), generator=g)))
    return sorted(rows)
