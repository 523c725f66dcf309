"""Sequence parallelism over several processes (sequence_head_attention_b200/dist.py) on CPU: gloo ranks
exchange real collectives, and the copies and attention launches are the oracle's (fp64), injected where
the GPU path calls the library's kernels.  What is checked is the exchange: which block goes where and
when, the all-to-all layout, the ring's schedule and its causal skips, and that the result is full
attention over the whole sequence ("HCMS", abstract: all-to-all sequence parallelism; "CHARM+: How
Cross-Hardware Attention ...", Ring-Attention paragraph)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleKernels:
    """fp64 stand-ins for the library's kernels on CPU tensors, built from the oracle."""
    acc_dtype = torch.float64

    @staticmethod
    def split_heads(x, outs, heads):
        import oracle
        h0, n = heads
        for o, part in zip(outs, oracle.split_heads(x.numpy(), len(outs))):
            o.copy_(torch.from_numpy(part[:, :, h0:h0 + n]))

    @staticmethod
    def merge_heads(ins, out, heads):
        # the stage's heads of each group into out (the oracle's merge of whole groups, with the other heads
        # of every group taken from out as it stands)
        import oracle
        h0, n = heads
        P = len(ins)
        groups = oracle.split_heads(out.numpy(), P)
        for r in range(P):
            groups[r][:, :, h0:h0 + n] = ins[r].numpy()
        out.copy_(torch.from_numpy(oracle.merge_heads(groups)))

    @staticmethod
    def attention_sharded(q_shards, k_shards, v_shards, o_shards, lse, head_chunks, causal):
        import oracle
        q, k, v = (torch.cat(list(t), dim=1).numpy() for t in (q_shards, k_shards, v_shards))
        o, l = oracle.attention(q, k, v, causal=causal, nthreads=1)
        Sl = q_shards[0].shape[1]
        for g, t in enumerate(o_shards):
            t.copy_(torch.from_numpy(o[:, g * Sl:(g + 1) * Sl]))
        lse.copy_(torch.from_numpy(l))

    @staticmethod
    def partial(q, k, v, o_acc, lse_acc, causal):
        import oracle
        o, l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal=causal, nthreads=1)
        o_acc.copy_(torch.from_numpy(o))
        lse_acc.copy_(torch.from_numpy(l))

    @staticmethod
    def partial_merge(q, k, v, o_acc, lse_acc, causal):
        import oracle
        o, l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal=causal, nthreads=1)
        mo, ml = oracle.merge([o_acc.numpy().copy(), o], [lse_acc.numpy().copy(), l])
        o_acc.copy_(torch.from_numpy(mo))
        lse_acc.copy_(torch.from_numpy(ml))

    @staticmethod
    def finish(o_acc, o):
        o.copy_(o_acc)


def _inputs(B, S, H, D, seed):
    from sequence_head_attention_b200 import synth
    q, k, v = synth.qkv(B, S, H, D, seed=seed, scale=0.5)
    return q.double(), k.double(), v.double()


def _worker(rank, world, port, scheme, causal, out, stages=1):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle
    from sequence_head_attention_b200 import dist as sp_dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, S, H, D = 2, 48 * world, 4 * world, 8
        q, k, v = _inputs(B, S, H, D, seed=world)
        Sl = S // world
        mine = [t[:, rank * Sl:(rank + 1) * Sl].contiguous() for t in (q, k, v)]
        ref_o, ref_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal=causal, nthreads=1)
        if scheme == "ulysses":
            sp = sp_dist.UlyssesAttention(B, S, H, D, head_chunks=[1, H - 1], causal=causal, dtype=torch.float64,
                                          kernels=OracleKernels, stages=stages)
            o = sp.forward(*mine)
            # the exchanges delivered exactly the seq -> head relayout of every tensor (bit for bit), stage by
            # stage
            for i, t in enumerate((q, k, v)):
                shards = [t[:, g * Sl:(g + 1) * Sl].numpy() for g in range(world)]
                want = oracle.seq_to_head(shards, H)[rank]
                got = torch.cat([torch.cat([sp.recv[c][g, i] for g in range(world)], dim=1)
                                 for c in range(len(sp.stages))], dim=2).numpy()
                assert np.array_equal(got, want)
            Hl = H // world
            lse_err = float(np.max(np.abs(sp.lse_heads().numpy() - ref_l[:, rank * Hl:(rank + 1) * Hl])))
            rounds = None
        else:
            sp = sp_dist.RingAttention(B, S, H, D, causal=causal, dtype=torch.float64, kernels=OracleKernels)
            o = sp.forward(*mine)
            lse_err = float(np.max(np.abs(sp.lse.numpy() - ref_l[:, :, rank * Sl:(rank + 1) * Sl])))
            rounds = sp.rounds
        o_err = float(np.max(np.abs(o.numpy() - ref_o[:, rank * Sl:(rank + 1) * Sl])))
        out.put((rank, o_err, lse_err, rounds))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,scheme,causal,stages", [
    (2, "ulysses", False, 1), (4, "ulysses", True, 1), (2, "ulysses", True, 3), (4, "ulysses", False, 2),
    (2, "ring", False, 1), (2, "ring", True, 1), (4, "ring", False, 1), (4, "ring", True, 1),
])
def test_sequence_parallel_schemes_on_gloo_ranks(world, scheme, causal, stages):
    """Ulysses in one exchange and in head-chunk stages (HCMS: the next stage's all-to-all posted before the
    current stage's attention), and the ring, on 2 and 4 ranks."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, scheme, causal, q, stages)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, o_err, lse_err, rounds in got:
        assert o_err < 1e-12 and lse_err < 1e-12, (rank, o_err, lse_err)
        if rounds is not None:
            # round s holds rank (rank - s) mod P's block; causal computes only blocks g <= rank
            assert [g for _, g, _ in rounds] == [(rank - s) % world for s in range(world)]
            done = [what for _, g, what in rounds]
            if causal:
                assert done == ["causal"] + ["full"] * rank + ["skipped"] * (world - 1 - rank)
            else:
                assert done == ["full"] * world
