"""Sequence parallelism over P processes, one per GPU: the Ulysses all-to-all and the KV ring with real
collectives (torch.distributed; NCCL over NVLink between GPUs), the library's kernels in between.

Both schemes start from the same placement: rank r holds positions [r S/P, (r+1) S/P) of Q, K and V, all
heads, as [B, S/P, H, D] tensors in its own GPU's memory, and ends with the same rows of O.

UlyssesAttention   ("HCMS: Head-Chunked Multi-Stream Pipeline ...", abstract: all-to-all based sequence
                   parallelism, heads processed in chunks so that communication overlaps computation;
                   "db-SP ...", abstract: parallelism along the head dimension as in Ulysses)
    Each rank's H/P heads are processed in `stages` head chunks (1: one exchange of everything).  Per stage:
    1. sp_split_heads cuts each of Q, K, V into P head groups (the stage's heads of each rank's group),
       written straight into the stage's send buffer [P, 3, B, S/P, n, D] (block r goes to rank r);
    2. an all-to-all: block g of the receive buffer holds rank g's positions of this rank's stage heads;
    3. sp_attn_fwd_seq_sharded attends those heads over the whole sequence, reading the P received blocks as
       its sequence shards and writing O into the P blocks of the stage's O send buffer;
    4. an all-to-all returns O's blocks to the ranks that own those positions;
    5. sp_merge_heads places the stage's heads of the P groups into this rank's O shard [B, S/P, H, D].
    The collectives are asynchronous: the all-to-all of stage c + 1 is posted before the attention of stage
    c and awaited after it, and each stage's O goes back while the next stage computes, so with NCCL the
    exchanges run beside the attention kernels.  The lse stays head-sharded: rank r's [B, H/P, S].

RingAttention      ("CHARM+: How Cross-Hardware Attention Breaks Through Distributed Communication
                   Bottlenecks", Ring-Attention paragraph: Q stays local while the KV blocks travel round a
                   ring of devices, each round's partial result accumulated; "CHARM+: ... Re-Merge ...",
                   abstract: re-merge)
    P rounds.  In round s rank r holds the KV block of rank g = (r - s) mod P and merges its partial into a
    running (O, lse) in the attention epilogue (sp_attn_fwd_partial for the first round,
    sp_attn_fwd_partial_merge after it), while the block it holds goes to rank r + 1 and the next one
    arrives from rank r - 1 (point-to-point sends posted before the round's attention, waited for after
    it, so the transfer overlaps the compute).  Causal: the rank's own block is the diagonal (a causal
    launch), blocks of earlier ranks are fully visible (non-causal launches) and blocks of later ranks are
    not visible at all (skipped).  After the last round the running O is rounded to bf16.

Every transfer lands in the receiving GPU's own memory before any kernel reads it: the kernels only
ever read local buffers (no peer pointers, no multicast).

The copies and attention launches go through a ``kernels`` object; by default the library's
(``LibraryKernels``).  The classes only allocate buffers, order the launches and issue the collectives.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import spattn


def rank_chunks(chunks, H, P):
    """Split a global head-chunk list at the rank boundaries (multiples of H/P).  Each rank gets the
    chunks inside its head range; a chunk that straddles a boundary is cut there."""
    Hl = H // P
    out = [[] for _ in range(P)]
    h0 = 0
    for c in chunks:
        a, e = h0, h0 + c
        while a < e:
            r = a // Hl
            cut = min(e, (r + 1) * Hl)
            out[r].append(cut - a)
            a = cut
        h0 = e
    return out


class LibraryKernels:
    """The library's kernels (CUDA, one GPU), as the schemes below call them."""

    acc_dtype = torch.float32

    @staticmethod
    def split_heads(x, outs, heads):
        spattn.sp_split_heads(x, outs, heads=heads)

    @staticmethod
    def merge_heads(ins, out, heads):
        spattn.sp_merge_heads(ins, out, heads=heads)

    @staticmethod
    def attention_sharded(q_shards, k_shards, v_shards, o_shards, lse, head_chunks, causal):
        spattn.sp_attn_fwd_seq_sharded(q_shards, k_shards, v_shards, o_shards, lse, head_chunks=head_chunks,
                                       causal=causal)

    @staticmethod
    def partial(q, k, v, o_acc, lse_acc, causal):
        spattn.sp_attn_fwd_partial(q, k, v, o_acc, lse_acc, 0, q.shape[1], causal=causal)

    @staticmethod
    def partial_merge(q, k, v, o_acc, lse_acc, causal):
        spattn.sp_attn_fwd_partial_merge(q, k, v, o_acc, lse_acc, 0, q.shape[1], causal=causal)

    @staticmethod
    def finish(o_acc, o):
        spattn.sp_convert_f32_to_bf16(o_acc, o)


def stage_bounds(n, stages):
    """Contiguous near-equal head chunks of n heads in `stages` stages (the first ones one larger)."""
    stages = max(1, min(int(stages), n))
    q, r = divmod(n, stages)
    cuts = [0]
    for c in range(stages):
        cuts.append(cuts[-1] + q + (1 if c < r else 0))
    return list(zip(cuts[:-1], cuts[1:]))


class UlyssesAttention:
    def __init__(self, B, S, H, D, head_chunks=None, causal=False, group=None, device=None, dtype=torch.bfloat16,
                 kernels=LibraryKernels, stages=1):
        self.group = group
        self.P = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        P = self.P
        if S % P or H % P:
            raise ValueError("S and H must be multiples of the number of ranks")
        self.B, self.S, self.H, self.D, self.Sl, self.Hl = B, S, H, D, S // P, H // P
        self.causal = causal
        self.kernels = kernels
        self.stages = stage_bounds(self.Hl, stages)
        # the model's head chunks, cut at the rank boundaries and then at the stage boundaries (they only
        # order the work within a launch: each stage's launch takes its part of this rank's chunk list)
        rank_chunk = rank_chunks(head_chunks or (H,), H, P)[self.rank]
        self.chunks = []
        for h0, h1 in self.stages:
            part, a = [], 0
            for c in rank_chunk:
                lo, hi = max(a, h0), min(a + c, h1)
                if hi > lo:
                    part.append(hi - lo)
                a += c
            self.chunks.append(part)
        self.send, self.recv, self.o_send, self.o_recv, self.lse = [], [], [], [], []
        for h0, h1 in self.stages:
            blk = (B, self.Sl, h1 - h0, D)
            self.send.append(torch.empty((P, 3) + blk, dtype=dtype, device=device))
            self.recv.append(torch.empty((P, 3) + blk, dtype=dtype, device=device))
            self.o_send.append(torch.empty((P,) + blk, dtype=dtype, device=device))
            self.o_recv.append(torch.empty((P,) + blk, dtype=dtype, device=device))
            self.lse.append(torch.empty((B, h1 - h0, S), dtype=kernels.acc_dtype, device=device))

    def forward(self, q, k, v, out=None, phase=None):
        """q, k, v: this rank's [B, S/P, H, D] shards.  Returns its [B, S/P, H, D] shard of O; the lse of this
        rank's heads is left in self.lse (one [B, n, S] tensor per stage).  phase(name, fn), if given, runs
        each part (to bracket it with timing events)."""
        P, n = self.P, len(self.stages)
        run = phase or (lambda name, fn: fn())

        def a2a(dst, src):
            return dist.all_to_all_single(dst, src, group=self.group, async_op=True)

        def split():
            for c, (h0, h1) in enumerate(self.stages):
                for i, x in enumerate((q, k, v)):
                    self.kernels.split_heads(x, [self.send[c][r, i] for r in range(P)], (h0, h1 - h0))

        run("split", split)
        pending = {0: a2a(self.recv[0], self.send[0])}
        back = []
        for c in range(n):
            if c + 1 < n:
                pending[c + 1] = a2a(self.recv[c + 1], self.send[c + 1])  # the next stage's heads travel now
            run("exchange", pending.pop(c).wait)
            rc, oc = self.recv[c], self.o_send[c]
            run("attn", lambda rc=rc, oc=oc, c=c: self.kernels.attention_sharded(
                [rc[g, 0] for g in range(P)], [rc[g, 1] for g in range(P)], [rc[g, 2] for g in range(P)],
                [oc[g] for g in range(P)], self.lse[c], self.chunks[c], self.causal))
            back.append(a2a(self.o_recv[c], self.o_send[c]))  # this stage's O goes back while the next computes
        o = out if out is not None else torch.empty_like(q)
        for c, (h0, h1) in enumerate(self.stages):
            run("exchange", back[c].wait)
            run("merge", lambda c=c, h0=h0, h1=h1: self.kernels.merge_heads(
                [self.o_recv[c][r] for r in range(P)], o, (h0, h1 - h0)))
        return o

    def lse_heads(self):
        """This rank's lse [B, H/P, S] (the stages' lse joined along the heads)."""
        return torch.cat(self.lse, dim=1)

    def bytes_exchanged(self):
        """Bytes this rank sends to other ranks per forward (Q, K, V out, O back; its own block stays)."""
        per_block = self.B * self.Sl * self.Hl * self.D * self.send[0].element_size()
        return 4 * (self.P - 1) * per_block


class RingAttention:
    def __init__(self, B, S, H, D, causal=False, group=None, device=None, dtype=torch.bfloat16,
                 kernels=LibraryKernels):
        self.group = group
        self.P = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if S % self.P:
            raise ValueError("S must be a multiple of the number of ranks")
        self.B, self.S, self.H, self.D, self.Sl = B, S, H, D, S // self.P
        self.causal = causal
        self.kernels = kernels
        shard = (B, self.Sl, H, D)
        # the KV blocks arriving from the ring, two slots (the first round uses the caller's K and V)
        self.k_in = [torch.empty(shard, dtype=dtype, device=device) for _ in range(2)]
        self.v_in = [torch.empty(shard, dtype=dtype, device=device) for _ in range(2)]
        self.o_acc = torch.empty(shard, dtype=kernels.acc_dtype, device=device)
        self.lse = torch.empty((B, H, self.Sl), dtype=kernels.acc_dtype, device=device)
        self.rounds = []  # (round, source rank, what was done) of the last forward

    def _peer(self, r):
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def forward(self, q, k, v, out=None, phase=None):
        """q, k, v: this rank's [B, S/P, H, D] shards.  Returns its [B, S/P, H, D] shard of O (its lse, natural
        log, is left in self.lse).  phase(name, fn), if given, runs each attention launch and the final
        rounding (to bracket them with timing events)."""
        run = phase or (lambda name, fn: fn())
        P, r = self.P, self.rank
        ck, cv = k, v
        self.rounds = []
        first = True
        for s in range(P):
            g = (r - s) % P  # the rank whose KV block this rank holds in round s
            nk, nv = self.k_in[s % 2], self.v_in[s % 2]
            reqs = []
            if s < P - 1:  # pass the block on while it is used
                nxt_rank, prev_rank = self._peer((r + 1) % P), self._peer((r - 1) % P)
                reqs = dist.batch_isend_irecv([
                    dist.P2POp(dist.isend, ck, nxt_rank, self.group), dist.P2POp(dist.isend, cv, nxt_rank, self.group),
                    dist.P2POp(dist.irecv, nk, prev_rank, self.group), dist.P2POp(dist.irecv, nv, prev_rank, self.group)])
            if self.causal and g > r:
                what = "skipped"  # every key of a later rank's block is after every query here
            else:
                diag = self.causal and g == r
                if first:
                    run("attn", lambda: self.kernels.partial(q, ck, cv, self.o_acc, self.lse, diag))
                    first = False
                else:
                    run("attn", lambda: self.kernels.partial_merge(q, ck, cv, self.o_acc, self.lse, diag))
                what = "causal" if diag else "full"
            self.rounds.append((s, g, what))
            for req in reqs:
                req.wait()
            ck, cv = nk, nv
        o = out if out is not None else torch.empty(q.shape, dtype=q.dtype, device=q.device)
        run("finish", lambda: self.kernels.finish(self.o_acc, o))
        return o

    def bytes_exchanged(self):
        """Bytes this rank sends per forward: a K and a V block in each of P - 1 rounds."""
        return (self.P - 1) * 2 * self.B * self.Sl * self.H * self.D * self.k_in[0].element_size()
