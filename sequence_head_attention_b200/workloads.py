"""The three full-size launch configurations, as steps the benchmark times and the tests check.

Each step owns its device buffers (allocated once with torch), and ``run()`` enqueues one pass of its
part of the path on the current stream through the C ABI; nothing here computes anything itself.

UlyssesStep   video-DiT shape: Q, K, V arrive as P sequence shards (one buffer per simulated rank);
              seq -> head relayout of each; attention of every rank on its H/P heads, with the global
              head chunks split at the rank boundaries; head -> seq relayout of O back to sequence shards.
              With fused=True each rank's attention reads the sequence shards and writes O into them
              directly (sp_attn_fwd_seq_sharded), with the same result and no relayout pass.
RingStep      long causal shape: 8 contiguous KV blocks, one launch each (every query against one block),
              the first writing the running fp32 result and every later one merging its rows into it in
              place (log-sum-exp rule), then the running O rounded to bf16.  The standalone re-merge of
              materialised partials (sp_merge_partials) is kept for its own measurement.
SparseStep    block-sparse DiT shape: tile-list build from the mask, then one attention launch that
              skips dropped tiles.
"""
from __future__ import annotations

import torch

from . import spattn
from .dist import rank_chunks  # noqa: F401  (the head chunks of each simulated rank)
from .synth import TILE, Workload, split_seq


class UlyssesStep:
    def __init__(self, w: Workload, q, k, v, device="cuda", fused=False):
        self.w = w
        self.fused = fused
        P, B, S, H, D = w.ranks, w.B, w.S, w.H, w.D
        self.P, self.Hl = P, H // P
        self.chunks = rank_chunks(w.head_chunks or (H,), H, P)
        self.q_seq = [t.to(device) for t in split_seq(q, P)]
        self.k_seq = [t.to(device) for t in split_seq(k, P)]
        self.v_seq = [t.to(device) for t in split_seq(v, P)]
        shard = (B, S, self.Hl, D)
        self.q_head = [torch.empty(shard, dtype=torch.bfloat16, device=device) for _ in range(P)]
        self.k_head = [torch.empty(shard, dtype=torch.bfloat16, device=device) for _ in range(P)]
        self.v_head = [torch.empty(shard, dtype=torch.bfloat16, device=device) for _ in range(P)]
        self.o_head = [torch.empty(shard, dtype=torch.bfloat16, device=device) for _ in range(P)]
        self.lse = [torch.empty((B, self.Hl, S), dtype=torch.float32, device=device) for _ in range(P)]
        self.o_seq = [torch.empty((B, S // P, H, D), dtype=torch.bfloat16, device=device) for _ in range(P)]
        self.lse_all = torch.empty((B, H, S), dtype=torch.float32, device=device)  # fused path
        self.launches = P if fused else 3 + P + 1
        self.flops = w.flops()
        self.relayout_bytes = 4 * 2 * B * S * H * D * 2  # 4 tensors, each read once and written once
        # one rank's attention launch: its heads of Q, K, V read and of O written (bf16), and its lse rows
        self.attn_bytes_per_launch = 4 * B * S * self.Hl * D * 2 + B * self.Hl * S * 4

    def relayout_in(self, stream=None):
        spattn.sp_seq_to_head_relayout(self.q_seq, self.q_head, stream=stream)
        spattn.sp_seq_to_head_relayout(self.k_seq, self.k_head, stream=stream)
        spattn.sp_seq_to_head_relayout(self.v_seq, self.v_head, stream=stream)

    def attention(self, stream=None):
        for r in range(self.P):
            spattn.sp_attn_fwd(self.q_head[r], self.k_head[r], self.v_head[r], self.o_head[r], self.lse[r],
                               head_chunks=self.chunks[r], stream=stream)

    def relayout_out(self, stream=None):
        spattn.sp_head_to_seq_relayout(self.o_head, self.o_seq, stream=stream)

    def attention_rank_fused(self, r, stream=None):
        spattn.sp_attn_fwd_seq_sharded(self.q_seq, self.k_seq, self.v_seq, self.o_seq, self.lse_all,
                                       heads=(r * self.Hl, self.Hl), head_chunks=self.chunks[r], stream=stream)

    def run(self, stream=None):
        if self.fused:
            for r in range(self.P):
                self.attention_rank_fused(r, stream)
            return
        self.relayout_in(stream)
        self.attention(stream)
        self.relayout_out(stream)

    def lse_full(self):
        return self.lse_all if self.fused else torch.cat(self.lse, dim=1)

    def inputs(self):
        return self.q_seq + self.k_seq + self.v_seq

    def outputs(self):
        return self.o_seq


class RingStep:
    def __init__(self, w: Workload, q, k, v, device="cuda", with_partials=False):
        self.w = w
        B, S, H, D = w.B, w.S, w.H, w.D
        self.q, self.k, self.v = q.to(device), k.to(device), v.to(device)
        n = w.n_kv_blocks
        self.blk = (S + n - 1) // n
        self.blocks = [(i * self.blk, min(S, (i + 1) * self.blk)) for i in range(n) if i * self.blk < S]
        self.o_acc = torch.empty((B, S, H, D), dtype=torch.float32, device=device)
        self.lse = torch.empty((B, H, S), dtype=torch.float32, device=device)
        self.o = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=device)
        self.attn_launches = len(self.blocks)
        self.launches = len(self.blocks) + 1  # the block launches and the bf16 rounding
        self.flops = w.flops()
        # the bf16 rounding of the running O: read fp32, write bf16
        self.convert_bytes = B * S * H * D * (4 + 2)
        # standalone re-merge of n materialised partials: read n fp32 partials (O and LSE), write bf16 O, fp32 LSE
        self.merge_bytes = n * (B * S * H * D * 4 + B * H * S * 4) + B * S * H * D * 2 + B * H * S * 4
        self.o_parts = self.l_parts = None
        if with_partials:
            self.o_parts = [torch.empty((B, S, H, D), dtype=torch.float32, device=device) for _ in range(n)]
            self.l_parts = [torch.empty((B, H, S), dtype=torch.float32, device=device) for _ in range(n)]
            self.o_merged = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=device)
            self.lse_merged = torch.empty((B, H, S), dtype=torch.float32, device=device)

    def attention(self, stream=None):
        """The ring's rounds: the first block's partial into the running result, later blocks merged in."""
        causal = self.w.causal
        a, e = self.blocks[0]
        spattn.sp_attn_fwd_partial(self.q, self.k, self.v, self.o_acc, self.lse, a, e, causal=causal, stream=stream)
        for a, e in self.blocks[1:]:
            spattn.sp_attn_fwd_partial_merge(self.q, self.k, self.v, self.o_acc, self.lse, a, e, causal=causal,
                                             stream=stream)

    def finish(self, stream=None):
        spattn.sp_convert_f32_to_bf16(self.o_acc, self.o, stream=stream)

    def run(self, stream=None):
        self.attention(stream)
        self.finish(stream)

    def partials(self, stream=None):
        """Every block's partial materialised (sp_attn_fwd_partial), the input of the standalone merge."""
        for i, (a, e) in enumerate(self.blocks):
            spattn.sp_attn_fwd_partial(self.q, self.k, self.v, self.o_parts[i], self.l_parts[i], a, e,
                                       causal=self.w.causal, stream=stream)

    def merge(self, stream=None):
        spattn.sp_merge_partials(self.o_parts, self.l_parts, self.o_merged, self.lse_merged, stream=stream)

    def workspace_for_fwd(self):
        w = self.w
        n = spattn.sp_attn_fwd_workspace_bytes(w.B, w.S, w.H, w.D, w.n_kv_blocks, False)
        return torch.empty(n, dtype=torch.uint8, device=self.q.device)

    def inputs(self):
        return [self.q, self.k, self.v]

    def outputs(self):
        return [self.o]


class SparseStep:
    def __init__(self, w: Workload, q, k, v, mask, device="cuda"):
        self.w = w
        B, S, H, D = w.B, w.S, w.H, w.D
        self.q, self.k, self.v = q.to(device), k.to(device), v.to(device)
        self.mask = mask.to(device)
        self.kept_tiles = int(mask.to(torch.int64).sum())
        self.density = self.kept_tiles / float(mask.numel())
        self.o = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((B, H, S), dtype=torch.float32, device=device)
        self.ws = torch.empty(spattn.sp_attn_fwd_workspace_bytes(B, S, H, D, 1, True), dtype=torch.uint8,
                              device=device)
        self.launches = 3 + 1
        # algorithmic FLOPs: 4 * D * 128 * 128 per kept tile and batch (QK^T and PV, 2 FLOPs per MAC)
        self.flops = 4.0 * B * D * TILE * TILE * self.kept_tiles

    def run(self, stream=None):
        spattn.sp_attn_fwd(self.q, self.k, self.v, self.o, self.lse, block_mask=self.mask,
                           workspace=self.ws, stream=stream)

    def rank_items(self, P: int, planned: bool):
        """Device item lists of P simulated sequence-parallel ranks: the db-SP two-level plan, or the
        contiguous head split of Ulysses (rank r takes heads [r H/P, (r+1) H/P)).  Returns (lists,
        imbalance ratio)."""
        import numpy as np
        w = self.w
        T = (w.S + TILE - 1) // TILE
        cost = spattn.sp_dbsp_unit_costs(self.mask.cpu(), w.H, T, w.causal)
        if planned:
            unit_rank, load, imb = spattn.sp_dbsp_plan(cost, P)
        else:
            unit_rank = np.repeat((np.arange(w.H) * P // w.H)[:, None], cost.shape[1], axis=1).astype(np.int32)
            load = np.array([cost[unit_rank == r].sum() for r in range(P)])
            imb = float(load.max() * P / load.sum())
        lists = [torch.from_numpy(spattn.sp_dbsp_rank_items(cost, unit_rank, w.B, r)).to(self.q.device)
                 for r in range(P)]
        return lists, imb

    def run_items(self, items, stream=None):
        spattn.sp_attn_fwd_items(self.q, self.k, self.v, self.o, self.lse, items, causal=self.w.causal,
                                 block_mask=self.mask, workspace=self.ws, stream=stream)

    def inputs(self):
        return [self.q, self.k, self.v]

    def outputs(self):
        return [self.o]
