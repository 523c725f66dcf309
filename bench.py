#!/usr/bin/env python
"""Benchmark of the sequence/head-parallel attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step is one pass of the path over one batch of synthetic input (inputs resident in HBM):

  video_dit (default)  B1 S32760 H40 D128, N(0,1)*0.5: Q, K, V as 4 sequence shards (simulated ranks);
                       seq->head relayout of each, attention of every rank on its 10 heads with the head
                       chunks [3,7,10,10,10] split at rank boundaries, head->seq relayout of O.
  ring_causal          B1 S57344 H40 D128 causal: 8 KV-block partial launches + log-sum-exp merge.
  block_sparse         B1 S32768 H40 D128, per-head tile mask of density U[0.1, 0.9]: tile list + attention.

The metric is attention TFLOPS (4 B H S^2 D x density, halved when causal) over the step time; the
relayout and merge GB/s are reported beside it under "kernels".  With N > 1 (torchrun, one rank per GPU)
every rank runs its own batch (weak scaling, no data-path collective); time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this path has) on the host cores, on a
bounded sample of the same workload, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention TFLOPS & % of bf16 tensor peak at S=32K–56K; relayout/merge GB/s"
UNIT = "TFLOPS"


# ----------------------------------------------------------------------------------------------------
# distributed plumbing (NCCL on GPUs, gloo on CPU); used by the tests with gloo
# ----------------------------------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str, timeout_s: int = 120):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish_dist():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


def emit(line: dict, rank: int):
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def recorded_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on the current
    kernel sources (their sha256 is recorded beside it); otherwise None."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", "attn_fwd_kernel_video_dit.md")
    try:
        text = open(path).read()
        h = hashlib.sha256()
        for f in ("attn_fwd.cu", "sp_ptx.cuh"):
            with open(os.path.join(ROOT, "sequence_head_attention_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
        sha = re.search(r"kernel_sources_sha256: ([0-9a-f]{64})", text).group(1)
        val = int(re.search(r"traffic_bytes_per_launch: (\d+)", text).group(1))
    except (OSError, AttributeError, ValueError):
        return None
    return val if sha == h.hexdigest() else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------------------------------
# CPU oracle timing (the cpu_baseline of our arm, and the whole of the reference arm)
# ----------------------------------------------------------------------------------------------------
def oracle_sample(wname: str, q, k, v, mask, n_rows: int, heads, seed: int = 0, w=None):
    """Run the fp64 oracle on n_rows sampled query rows of the given heads; return (seconds, flops,
    threads, description).  FLOPs are counted like the metric: 4 * D per (row, visible key)."""
    import numpy as np
    import oracle
    from sequence_head_attention_b200 import synth
    w = w or synth.WORKLOADS[wname]
    rows = synth.sample_rows(w.S, n_rows, seed=seed)[:n_rows]
    hs = list(heads)
    q64 = q[:, :, hs][:, rows].double().numpy()
    k64 = k[:, :, hs].double().numpy()
    v64 = v[:, :, hs].double().numpy()
    m = None if mask is None else mask[hs].numpy()
    # the oracle evaluates the chosen rows against all keys; Q is passed full-length with only the
    # sampled rows filled in, so row indices keep their global positions
    qfull = np.zeros((w.B, w.S, len(hs), w.D))
    qfull[:, rows] = q64
    nthreads = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.attention(qfull, k64, v64, causal=w.causal, block_mask=m, rows=rows, nthreads=nthreads)
    dt = time.perf_counter() - t0
    if mask is not None:
        keys = sum(int(mask[h, r // synth.TILE].sum()) * synth.TILE for h in hs for r in rows)
    elif w.causal:
        keys = sum(r + 1 for r in rows) * len(hs)
    else:
        keys = w.S * len(rows) * len(hs)
    flops = 4.0 * w.D * keys * w.B
    desc = f"{len(rows)} stratified query rows x {len(hs)} heads of {wname} (all keys), fp64"
    return dt, flops, nthreads, desc


def calibrated_oracle_baseline(wname, q, k, v, mask, target_s=15.0):
    heads = list(range(0, q.shape[2], 5))[:8]
    dt1, _, _, _ = oracle_sample(wname, q, k, v, mask, 4, heads)
    n = int(max(4, min(2048, 4 * target_s / max(dt1, 1e-3))))
    dt, flops, nthreads, desc = oracle_sample(wname, q, k, v, mask, n, heads)
    if dt < 0.5 * target_s and n < 2048:  # the 4-row probe overstates the per-row time (thread start-up)
        n = int(max(4, min(2048, n * target_s / max(dt, 1e-3))))
        dt, flops, nthreads, desc = oracle_sample(wname, q, k, v, mask, n, heads)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": desc, "seconds": round(dt, 3)}


# ----------------------------------------------------------------------------------------------------
def build_inputs(wname: str, seed: int, seq_len: int = 0, ranks: int = 0):
    import dataclasses
    from sequence_head_attention_b200 import synth
    w = synth.WORKLOADS[wname]
    if seq_len:
        w = dataclasses.replace(w, S=seq_len)
    if ranks:
        w = dataclasses.replace(w, ranks=ranks)
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=seed, scale=w.scale)
    mask = synth.block_mask(w.H, w.S, seed=seed) if w.sparse else None
    return w, q, k, v, mask


def config_of(w, wname, world, extra=None):
    c = {"workload": f"{wname}: B{w.B} S{w.S} H{w.H} D{w.D}" + (" causal" if w.causal else ""),
         "global_batch": w.B * world, "seq_len": w.S, "heads": w.H, "head_dim": w.D,
         "parallelism": f"replicas{world}" if world > 1 else "single",
         "l2": "inputs larger than L2 (Q, K, V >= 335 MB each); no flush"}
    if wname == "video_dit":
        c.update({"head_chunks": list(w.head_chunks), "simulated_ranks": w.ranks})
    if wname == "ring_causal":
        c.update({"kv_blocks": w.n_kv_blocks})
    if extra:
        c.update(extra)
    return c


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0  # the CPU oracle runs once, on rank 0
    w, q, k, v, mask = build_inputs(args.workload, seed=0)
    heads = list(range(0, w.H, 5))[:8]
    n_rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(args.workload, q, k, v, mask, n_rows, heads)
    times, flops_total = [], 0.0
    desc, nthreads = "", 1
    for _ in range(args.steps):
        dt, flops, nthreads, desc = oracle_sample(args.workload, q, k, v, mask, n_rows, heads)
        times.append(dt)
        flops_total += flops
    total = sum(times)
    value = flops_total / total / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * total / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args.workload, 1), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    emit(line, 0)
    return 0


def backward_report(w, q, k, v, reps, stream, E, peaks, dev):
    """The backward pass (sp_attn_bwd: delta, dK/dV and dQ launches) on one simulated rank's heads of the
    workload (heads 0 .. H/P - 1, all S positions), timed with CUDA events after the timed region.
    Algorithmic FLOPs: 10 B H S^2 D (five S x S x D products; halved when causal)."""
    import torch
    from sequence_head_attention_b200 import spattn
    hl = w.H // max(1, w.ranks)
    qh, kh, vh = (t[:, :, :hl].contiguous().to(dev) for t in (q, k, v))
    B, S, _, D = qh.shape
    o = torch.empty_like(qh)
    lse = torch.empty((B, hl, S), dtype=torch.float32, device=dev)
    spattn.sp_attn_fwd(qh, kh, vh, o, lse, causal=w.causal)
    do = torch.randn(qh.shape, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).to(dev)
    dq, dk, dv = (torch.empty_like(qh) for _ in range(3))
    ws = torch.empty(spattn.lib().sp_attn_bwd_workspace_bytes(B, S, hl, D), dtype=torch.uint8, device=dev)
    for _ in range(2):
        spattn.sp_attn_bwd(qh, kh, vh, o, do, lse, dq, dk, dv, causal=w.causal, workspace=ws)
    torch.cuda.synchronize(dev)
    a = E(); a.record(stream)
    for _ in range(reps):
        spattn.sp_attn_bwd(qh, kh, vh, o, do, lse, dq, dk, dv, causal=w.causal, workspace=ws)
    b = E(); b.record(stream)
    torch.cuda.synchronize(dev)
    if spattn.sp_check_device_error() != spattn.SP_OK:
        raise SystemExit("device error in the backward pass")
    ms = a.elapsed_time(b) / reps
    flops = 10.0 * B * hl * S * S * D / (2.0 if w.causal else 1.0)
    tf = flops / (ms / 1000.0) / 1e12
    return {"shape": f"B{B} S{S} H{hl} D{D}" + (" causal" if w.causal else ""), "ms": ms, "tflops": tf,
            "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"], "launches": 3,
            "flops_counted": "10 B H S^2 D (5 matrix products); the kernels execute 7 (S and dP are recomputed for dQ)"}


def dbsp_ranks_report(step, P, reps, stream, E):
    """Block-sparse attention split over P simulated sequence-parallel ranks, by the contiguous head split
    of Ulysses and by the db-SP plan: each rank's item-list launch is timed on its own (CUDA events), and
    a parallel step would take the slowest rank's time."""
    import torch
    out = {"ranks": P, "how": "per-rank item-list launches timed one by one on this GPU; step = slowest rank"}
    for name, planned in (("head_split", False), ("planned", True)):
        lists, imb = step.rank_items(P, planned)
        for items in lists:  # warm-up
            step.run_items(items)
        marks = []
        for _ in range(reps):
            for r, items in enumerate(lists):
                a = E(); a.record(stream); step.run_items(items); b = E(); b.record(stream)
                marks.append((r, a, b))
        torch.cuda.synchronize()
        per_rank = [statistics.mean(a.elapsed_time(b) for rr, a, b in marks if rr == r) for r in range(P)]
        out[name] = {"imbalance": imb, "rank_ms": per_rank, "max_rank_ms": max(per_rank)}
    out["speedup_of_plan"] = out["head_split"]["max_rank_ms"] / out["planned"]["max_rank_ms"]
    return out


def run_ours(args):
    import torch
    from sequence_head_attention_b200 import spattn, workloads

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl", timeout_s=180)
    spattn.lib()  # fail now if the library is missing

    w, q, k, v, mask = build_inputs(args.workload, seed=rank, seq_len=args.seq_len, ranks=args.ranks)
    fused = args.workload == "video_dit" and args.ulysses == "fused"
    if args.workload == "video_dit":
        step = workloads.UlyssesStep(w, q, k, v, device=dev, fused=fused)
    elif args.workload == "ring_causal":
        step = workloads.RingStep(w, q, k, v, device=dev)
    else:
        step = workloads.SparseStep(w, q, k, v, mask, device=dev)
    stream = torch.cuda.current_stream(dev)
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def timed_step(marks):
        """One step with events around the phases: returns nothing; marks collects (name, ev0, ev1)."""
        if fused:
            for r in range(step.P):
                a = E(); a.record(stream); step.attention_rank_fused(r); b = E(); b.record(stream)
                marks.append(("attn", a, b))
        elif args.workload == "video_dit":
            a = E(); a.record(stream); step.relayout_in(); b = E(); b.record(stream)
            marks.append(("relayout", a, b))
            for r in range(step.P):
                a = E(); a.record(stream)
                spattn.sp_attn_fwd(step.q_head[r], step.k_head[r], step.v_head[r], step.o_head[r], step.lse[r],
                                   head_chunks=step.chunks[r])
                b = E(); b.record(stream)
                marks.append(("attn", a, b))
            a = E(); a.record(stream); step.relayout_out(); b = E(); b.record(stream)
            marks.append(("relayout", a, b))
        elif args.workload == "ring_causal":
            a = E(); a.record(stream); step.attention(); b = E(); b.record(stream)
            marks.append(("attn_all", a, b))
            a = E(); a.record(stream); step.merge(); b = E(); b.record(stream)
            marks.append(("merge", a, b))
        else:
            a = E(); a.record(stream); step.run(); b = E(); b.record(stream)
            marks.append(("attn", a, b))

    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize(dev)
    if spattn.sp_check_device_error() != spattn.SP_OK:
        raise SystemExit("device error during warm-up")

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    marks = []
    t_start, t_end = E(), E()
    t_start.record(stream)
    for _ in range(args.steps):
        timed_step(marks)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    if spattn.sp_check_device_error() != spattn.SP_OK:
        raise SystemExit("device error during the timed steps")
    ms_local = t_start.elapsed_time(t_end)
    ms = max_over_ranks(ms_local, device=dev)
    total_flops = step.flops * args.steps * world
    value = total_flops / (ms / 1000.0) / 1e12

    peaks = measured_peaks()
    phase = {}
    for name, a, b in marks:
        phase.setdefault(name, []).append(a.elapsed_time(b))
    kernels = {}
    if args.workload == "video_dit":
        attn_ms = statistics.mean(phase["attn"])
        flops_launch = step.flops / step.P
        if not args.no_backward:
            kernels["backward"] = backward_report(w, q, k, v, max(3, args.steps // 2), stream, E, peaks, dev)
        if fused:
            # The fused step has no relayout pass; the relayout kernels (the unfused path's copies) are
            # timed here on their own, after the timed region, for their HBM figures.
            rl = []
            for _ in range(args.steps):
                a = E(); a.record(stream); step.relayout_in(); step.relayout_out(); b = E(); b.record(stream)
                rl.append((a, b))
            torch.cuda.synchronize(dev)
            rl_ms = statistics.mean(x.elapsed_time(y) for x, y in rl)
        else:
            rl_ms = sum(phase["relayout"]) / args.steps  # both relayout phases of one step
        rl_gbs = step.relayout_bytes / (rl_ms / 1000.0) / 1e9
        kernels["relayout"] = {"gbs": rl_gbs, "ms_per_step": rl_ms, "bytes_per_step": step.relayout_bytes,
                               "frac_of_measured_hbm": rl_gbs / peaks["hbm_gbs"],
                               "in_timed_step": not fused}
    elif args.workload == "ring_causal":
        attn_ms = statistics.mean(phase["attn_all"])
        flops_launch = step.flops
        m_ms = statistics.mean(phase["merge"])
        kernels["merge"] = {"gbs": step.merge_bytes / (m_ms / 1000.0) / 1e9, "ms": m_ms,
                            "bytes": step.merge_bytes,
                            "frac_of_measured_hbm": step.merge_bytes / (m_ms / 1000.0) / 1e9 / peaks["hbm_gbs"]}
    else:
        attn_ms = statistics.mean(phase["attn"])
        flops_launch = step.flops
        if args.dbsp_ranks > 1:
            kernels["dbsp"] = dbsp_ranks_report(step, args.dbsp_ranks, max(3, args.steps // 2), stream, E)
    achieved = flops_launch / (attn_ms / 1000.0) / 1e12
    kernels["attention"] = {"tflops": achieved, "ms_per_launch": attn_ms}
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops_sustained"],
                "traffic": recorded_traffic() if args.workload == "video_dit" and not args.seq_len and not args.ranks else None,
                "traffic_unit": "bytes per launch (dram read + write, ncu, profiles/attn_fwd_kernel_video_dit.md)",
                "peak_kind": f"{peaks['source']} bf16 dense, sustained (kernel timed inside a long step)",
                "frac_of_burst_peak": achieved / peaks["bf16_tflops"]}

    # End to end: every step's inputs come from pinned host memory and its O goes back to pinned host memory,
    # inside the timed region.  A second step object gives the pipeline its second slot, so the copies of
    # one step overlap the kernels of its neighbours (sequence_head_attention_b200/pipeline.py).
    e2e = None
    if not args.no_e2e:
        from sequence_head_attention_b200.pipeline import HostPipeline
        if args.workload == "video_dit":
            step2 = workloads.UlyssesStep(w, q, k, v, device=dev, fused=fused)
        elif args.workload == "ring_causal":
            step2 = workloads.RingStep(w, q, k, v, device=dev)
        else:
            step2 = workloads.SparseStep(w, q, k, v, mask, device=dev)
        slots = [step, step2]
        h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in step.inputs()]
        for h, t in zip(h_in, step.inputs()):
            h.copy_(t)
        h_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in s.outputs()] for s in slots]
        pipe = HostPipeline(slots, h_in, h_out)
        h2d, d2h = pipe.bytes_per_step()
        n_e2e = max(4, args.steps)
        pipe.run(2)  # warm the streams and the second slot
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        a = E(); a.record(stream)
        pipe.run(n_e2e, stream)
        b = E(); b.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        if spattn.sp_check_device_error() != spattn.SP_OK:
            raise SystemExit("device error during the end-to-end steps")
        e_ms = max_over_ranks(a.elapsed_time(b), device=dev)
        e2e = {"value": step.flops * n_e2e * world / (e_ms / 1000.0) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": e_ms / n_e2e,
               "pipeline": "2 step slots; H2D, kernels and D2H on three streams, overlapped across steps"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = calibrated_oracle_baseline(args.workload, q, k, v, mask, target_s=args.cpu_seconds)

    extra = {}
    if args.workload == "video_dit":
        extra = {"ulysses": "attention on the sequence shards, relayouts folded into the kernel" if fused
                 else "seq->head relayout, per-rank attention, head->seq relayout"}
    if args.workload == "block_sparse":
        extra = {"mask_density": step.density, "kept_tiles": step.kept_tiles}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, args.workload, world, extra), "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": step.launches * args.steps, "clocks": clocks, "kernels": kernels,
            "impl": "ours"}
    emit(line, rank)
    del step
    finish_dist()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["video_dit", "ring_causal", "block_sparse", "tiny_dense", "megatron"],
                    default="video_dit", help="tiny_dense / megatron: reference arm only (parity-size cases)")
    ap.add_argument("--ulysses", choices=["fused", "relayout"], default="fused",
                    help="video_dit step: attention straight on the sequence shards (fused), or the seq->head "
                         "relayout, per-rank attention and head->seq relayout")
    ap.add_argument("--dbsp-ranks", type=int, default=4,
                    help="block_sparse: also time the work split over this many simulated ranks, head split "
                         "vs db-SP plan (0: off)")
    ap.add_argument("--no-backward", action="store_true", help="video_dit: skip the backward-pass measurement")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=16, help="query rows per reference step")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override S (profiling captures on a smaller case; not a benchmark number)")
    ap.add_argument("--ranks", type=int, default=0,
                    help="override the simulated rank count of video_dit (profiling captures only)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload not in ("video_dit", "ring_causal", "block_sparse"):
        ap.error("--impl ours times the full-size workloads only")
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
