#!/usr/bin/env python
"""Benchmark of the sequence/head-parallel attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME|all]

One step is one pass of the path over one batch of synthetic input (inputs resident in HBM).  The default
(--workload all) prints ONE line headed by the S = 32K configuration and measures every other configuration
in the same run, each with its own CUDA-event timing and roofline block under "kernels":

  video_dit (headline)  B1 S32760 H40 D128, N(0,1)*0.5: Q, K, V as 4 sequence shards (simulated Ulysses
                        ranks); every rank's attention on its 10 heads with the head chunks [3,7,10,10,10]
                        split at rank boundaries, read from and written into the shards.  Also measured: the
                        seq<->head relayouts on their own (HBM GB/s) and the backward of one rank's heads.
  ring_causal           B1 S57344 H40 D128 causal: 8 KV blocks, one launch each; the first writes the running
                        (O, LSE), each later one merges its partial into it in place, and the running O is
                        rounded to bf16 (attention TFLOPS, step time).  The standalone re-merge of 8
                        materialised partials (sp_merge_partials) is timed on its own (merge GB/s).
  block_sparse          B1 S32768 H40 D128, per-head tile mask of density U[0.1, 0.9]: tile list +
                        attention (TFLOPS on kept tiles), and the db-SP split over 4 simulated ranks.
  tiny_dense, megatron  the two latency configurations: microseconds per call and TFLOPS, back to back
                        through the C ABI and replayed from a CUDA graph.

The metric is attention TFLOPS (4 B H S^2 D x density, halved when causal) over the step time.  Every
fraction of peak is taken against the measured burst bf16 GEMM rate (MEASURED_PEAKS.json): each timed
region here lasts well under a second.  With N > 1 (torchrun, one rank per GPU) every rank runs its own
batch (weak scaling, no data-path collective); the headline time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this path has) on the host cores, on a
bounded sample of the same workload, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention TFLOPS & % of bf16 tensor peak at S=32K–56K; relayout/merge GB/s"
UNIT = "TFLOPS"
ALL_WORKLOADS = ("video_dit", "ring_causal", "block_sparse", "tiny_dense", "megatron")
# DRAM traffic per launch from ncu captures (a plain data record kept beside the profile summaries)
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")


# ----------------------------------------------------------------------------------------------------
# distributed plumbing (NCCL on GPUs, gloo on CPU); used by the tests with gloo
# ----------------------------------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str, timeout_s: int = 120, always: bool = False):
    """Join the process group (torchrun's environment) when there are several ranks, or always (a group of
    one without torchrun, so that code issuing collectives also runs on a single GPU)."""
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if dist.is_initialized():
        return rank, world
    if world > 1 or (always and "MASTER_ADDR" in os.environ):
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    elif always:
        import socket
        with socket.socket() as s:
            s.bind(("127.0.0.1", 0))
            port = s.getsockname()[1]
        dist.init_process_group(backend=backend, init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=timeout_s))
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
# clocks during a timed region
# ----------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return parse_clock_rows(out)


def parse_clock_rows(out: str):
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


# ----------------------------------------------------------------------------------------------------
# peaks and recorded DRAM traffic
# ----------------------------------------------------------------------------------------------------
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


def sources_sha256(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "sequence_head_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(key: str):
    """(bytes per launch, note) for a kernel from the ncu traffic record, or (None, why not).  A figure is
    used only while the kernel's sources hash to the value recorded with it."""
    try:
        with open(TRAFFIC_RECORD) as f:
            entry = json.load(f)["entries"][key]
        if sources_sha256(entry["sources"]) != entry["sources_sha256"]:
            return None, "kernel changed since the ncu capture"
        note = entry.get("how", "ncu dram__bytes_read.sum + dram__bytes_write.sum")
        return int(entry["bytes_per_launch"]), note
    except (OSError, KeyError, ValueError, TypeError):
        return None, "no ncu capture recorded"


def tensor_roofline(flops_per_launch: float, ms_per_launch: float, peaks, traffic_key=None, algo_bytes=None):
    achieved = flops_per_launch / (ms_per_launch / 1000.0) / 1e12
    traffic, note = recorded_traffic(traffic_key) if traffic_key else (None, "not captured")
    r = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
         "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
         "peak_kind": f"{peaks['source']} bf16 dense GEMM, burst (timed regions here last well under a second)",
         "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
         "flops_per_launch": flops_per_launch, "ms_per_launch": ms_per_launch,
         "traffic_note": "bytes per launch (dram read + write, ncu): " + note}
    if algo_bytes is not None:
        r["algorithmic_bytes_per_launch"] = algo_bytes
    return r


def hbm_roofline(bytes_per_launch: float, ms_per_launch: float, peaks, traffic_key=None):
    achieved = bytes_per_launch / (ms_per_launch / 1000.0) / 1e9
    traffic, note = recorded_traffic(traffic_key) if traffic_key else (None, "not captured")
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "peak_kind": f"{peaks['source']} HBM copy bandwidth", "bytes_per_launch": bytes_per_launch,
            "ms_per_launch": ms_per_launch, "traffic_note": "bytes per launch (dram read + write, ncu): " + note}


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
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=seed, scale=w.scale, fp32_source=False)
    mask = synth.block_mask(w.H, w.S, seed=seed) if w.sparse else None
    return w, q, k, v, mask


def workload_name(w, wname):
    return f"{wname}: B{w.B} S{w.S} H{w.H} D{w.D}" + (" causal" if w.causal else "")


def config_of(w, wname, world, extra=None):
    c = {"workload": workload_name(w, wname), "global_batch": w.B * world, "seq_len": w.S, "heads": w.H,
         "head_dim": w.D, "parallelism": f"replicas{world}" if world > 1 else "single",
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
    wname = "video_dit" if args.workload == "all" else args.workload
    w, q, k, v, mask = build_inputs(wname, seed=0)
    heads = list(range(0, w.H, 5))[:8]
    n_rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(wname, q, k, v, mask, n_rows, heads)
    times, flops_total = [], 0.0
    desc, nthreads = "", 1
    for _ in range(args.steps):
        dt, flops, nthreads, desc = oracle_sample(wname, q, k, v, mask, n_rows, heads)
        times.append(dt)
        flops_total += flops
    total = sum(times)
    value = flops_total / total / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * total / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, wname, 1), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    emit(line, 0)
    return 0


# ----------------------------------------------------------------------------------------------------
# GPU measurements
# ----------------------------------------------------------------------------------------------------
class Timer:
    """CUDA events on one stream: phase(name) brackets a callable; mean_ms(name) averages its spans."""

    def __init__(self, stream):
        import torch
        self.stream = stream
        self.E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        self.marks = []

    def phase(self, name, fn):
        a = self.E(); a.record(self.stream)
        fn()
        b = self.E(); b.record(self.stream)
        self.marks.append((name, a, b))

    def spans(self, name):
        return [a.elapsed_time(b) for n, a, b in self.marks if n == name]

    def mean_ms(self, name):
        return statistics.mean(self.spans(name))


def check_device(where):
    from sequence_head_attention_b200 import spattn
    st, bits = spattn.sp_check_device_error_bits()
    if st != spattn.SP_OK:
        raise SystemExit(f"device error {spattn.sp_status_string(st)} (bits {bits:#x}) {where}")


def make_step(wname, w, q, k, v, mask, dev, fused=True, with_partials=False):
    from sequence_head_attention_b200 import workloads
    if wname == "video_dit":
        return workloads.UlyssesStep(w, q, k, v, device=dev, fused=fused)
    if wname == "ring_causal":
        return workloads.RingStep(w, q, k, v, device=dev, with_partials=with_partials)
    return workloads.SparseStep(w, q, k, v, mask, device=dev)


def step_phases(wname, step, fused, timer: Timer):
    """Enqueue one step with events around its phases."""
    from sequence_head_attention_b200 import spattn
    if wname == "video_dit" and fused:
        for r in range(step.P):
            timer.phase("attn", lambda r=r: step.attention_rank_fused(r))
    elif wname == "video_dit":
        timer.phase("relayout", step.relayout_in)
        for r in range(step.P):
            timer.phase("attn", lambda r=r: spattn.sp_attn_fwd(step.q_head[r], step.k_head[r], step.v_head[r],
                                                               step.o_head[r], step.lse[r],
                                                               head_chunks=step.chunks[r]))
        timer.phase("relayout", step.relayout_out)
    elif wname == "ring_causal":
        timer.phase("attn_all", step.attention)
        timer.phase("finish", step.finish)
    else:
        timer.phase("attn", step.run)


def backward_report(w, q, k, v, reps, stream, peaks, dev):
    """The backward pass (sp_attn_bwd: delta, dK/dV and dQ launches) on one simulated rank's heads of the
    workload (heads 0 .. H/P - 1, all S positions), timed with CUDA events.
    Algorithmic FLOPs: 10 B H S^2 D (five S x S x D products; halved when causal)."""
    import torch
    from sequence_head_attention_b200 import spattn
    hl = w.H // max(1, w.ranks)
    spattn.sp_set_launch_overlap(0)
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
    t = Timer(stream)
    for _ in range(reps):
        t.phase("bwd", lambda: spattn.sp_attn_bwd(qh, kh, vh, o, do, lse, dq, dk, dv, causal=w.causal, workspace=ws))
    torch.cuda.synchronize(dev)
    check_device("in the backward pass")
    ms = t.mean_ms("bwd")
    flops = 10.0 * B * hl * S * S * D / (2.0 if w.causal else 1.0)
    return {"shape": f"B{B} S{S} H{hl} D{D}" + (" causal" if w.causal else ""), "ms": ms,
            "tflops": flops / (ms / 1000.0) / 1e12, "launches": 3,
            "roofline": tensor_roofline(flops, ms, peaks),
            "flops_counted": "10 B H S^2 D (5 matrix products); the kernels execute 7 (S and dP are recomputed for dQ)"}


def dbsp_ranks_report(step, P, reps, stream):
    """Block-sparse attention split over P simulated sequence-parallel ranks, by the contiguous head split
    of Ulysses and by the db-SP plan: each rank's item-list launch is timed on its own (CUDA events), and
    a parallel step would take the slowest rank's time."""
    import torch
    out = {"ranks": P, "how": "per-rank item-list launches timed one by one on this GPU; step = slowest rank"}
    for name, planned in (("head_split", False), ("planned", True)):
        lists, imb = step.rank_items(P, planned)
        for items in lists:  # warm-up
            step.run_items(items)
        t = Timer(stream)
        for _ in range(reps):
            for r, items in enumerate(lists):
                t.phase(r, lambda items=items: step.run_items(items))
        torch.cuda.synchronize()
        per_rank = [t.mean_ms(r) for r in range(P)]
        out[name] = {"imbalance": imb, "rank_ms": per_rank, "max_rank_ms": max(per_rank)}
    out["speedup_of_plan"] = out["head_split"]["max_rank_ms"] / out["planned"]["max_rank_ms"]
    return out


def relayout_report(step, reps, stream, peaks):
    """The seq->head relayouts of Q, K, V and the head->seq relayout of O (the Ulysses exchange on one GPU),
    timed on their own; per-launch roofline of the seq->head kernel."""
    import torch
    step.relayout_in(); step.relayout_out()
    torch.cuda.synchronize()
    t = Timer(stream)
    for _ in range(reps):
        t.phase("pair", lambda: (step.relayout_in(), step.relayout_out()))
    for _ in range(reps):
        t.phase("one", lambda: spattn_relayout_one(step))
    torch.cuda.synchronize()
    check_device("in the relayouts")
    ms = t.mean_ms("pair")
    per_launch = step.relayout_bytes / 4  # one tensor: read and written once
    gbs = step.relayout_bytes / (ms / 1000.0) / 1e9
    return {"gbs": gbs, "ms_per_step": ms, "bytes_per_step": step.relayout_bytes, "launches_per_step": 4,
            "frac_of_measured_hbm": gbs / peaks["hbm_gbs"],
            "roofline": hbm_roofline(per_launch, t.mean_ms("one"), peaks, "relayout_seq_to_head.video_dit")}


def spattn_relayout_one(step):
    from sequence_head_attention_b200 import spattn
    spattn.sp_seq_to_head_relayout(step.q_seq, step.q_head)


def clock_sampler(dev):
    import torch
    return ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))


def measure_main(wname, args, peaks, dev, stream, world, seed, headline):
    """Time one full-size workload: W warm-up steps, then K steps between barrier + synchronize, CUDA events
    on the launching stream, max over ranks.  Returns (record, step, inputs)."""
    import torch
    from sequence_head_attention_b200 import spattn
    w, q, k, v, mask = build_inputs(wname, seed=seed, seq_len=args.seq_len if headline else 0,
                                    ranks=args.ranks if headline else 0)
    fused = wname == "video_dit" and args.ulysses == "fused"
    # Launch overlap where the step's attention launches follow one another and no kernel writes the Q, K, V
    # of the launch after it: the per-rank launches on the shards, the ring's blocks, the masked launches.
    # The per-rank launches also write disjoint heads of the shards (and lse rows), so they overlap their
    # outputs too (mode 2); a ring block reads the running result the block before wrote (mode 1).
    overlap = 0 if args.no_overlap or (wname == "video_dit" and not fused) else (2 if fused else 1)
    spattn.sp_set_launch_overlap(overlap)
    step = make_step(wname, w, q, k, v, mask, dev, fused, with_partials=wname == "ring_causal")
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize(dev)
    check_device(f"during the {wname} warm-up")
    sampler = clock_sampler(dev).start()
    barrier()
    torch.cuda.synchronize(dev)
    timer = Timer(stream)
    t_start, t_end = timer.E(), timer.E()
    t_start.record(stream)
    for _ in range(args.steps):
        step_phases(wname, step, fused, timer)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    check_device(f"during the {wname} timed steps")
    ms = max_over_ranks(t_start.elapsed_time(t_end), device=dev)
    value = step.flops * args.steps * world / (ms / 1000.0) / 1e12
    rec = {"workload": workload_name(w, wname), "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ms / args.steps, "tflops": value, "launches_per_step": step.launches, "clocks": clocks,
           "launch_overlap": overlap}
    if wname == "video_dit":
        attn_ms = timer.mean_ms("attn")
        rec["attention"] = {"tflops": step.flops / step.P / (attn_ms / 1000.0) / 1e12, "ms_per_launch": attn_ms,
                            "launches_per_step": step.P,
                            "roofline": tensor_roofline(step.flops / step.P, attn_ms, peaks,
                                                        "attn_fwd.video_dit_rank" if fused and not args.seq_len
                                                        and not args.ranks else None,
                                                        algo_bytes=step.attn_bytes_per_launch)}
        if not fused:
            rec["relayout_in_step_ms"] = sum(timer.spans("relayout")) / args.steps
    elif wname == "ring_causal":
        attn_ms = timer.mean_ms("attn_all")
        f_ms = timer.mean_ms("finish")
        rec["attention"] = {"tflops": step.flops / (attn_ms / 1000.0) / 1e12, "ms_per_step": attn_ms,
                            "launches_per_step": step.attn_launches,
                            "how": "first KV block written, every later block merged into the running result "
                                   "in its epilogue (sp_attn_fwd_partial_merge); no partial is materialised",
                            "roofline": tensor_roofline(step.flops, attn_ms, peaks, None)}
        rec["attention"]["roofline"]["traffic_note"] = ("the attention of a ring step is several launches; "
                                                        "traffic per launch is not recorded")
        rec["finish"] = {"what": "running fp32 O rounded to bf16", "ms": f_ms,
                         "gbs": step.convert_bytes / (f_ms / 1000.0) / 1e9}
        rec["merge"] = merge_report(step, args, peaks, stream)
    else:
        attn_ms = timer.mean_ms("attn")
        rec["attention"] = {"tflops": step.flops / (attn_ms / 1000.0) / 1e12, "ms_per_launch": attn_ms,
                            "roofline": tensor_roofline(step.flops, attn_ms, peaks,
                                                        "attn_fwd.block_sparse" if not args.seq_len else None),
                            "mask_density": step.density, "kept_tiles": step.kept_tiles}
    return rec, step, (w, q, k, v, mask, fused)


def merge_report(step, args, peaks, stream):
    """The standalone re-merge (sp_merge_partials) of the ring's 8 materialised fp32 partials into bf16 O and
    fp32 LSE, timed on its own after the timed steps."""
    import torch
    step.partials()
    step.merge()
    torch.cuda.synchronize()
    t = Timer(stream)
    for _ in range(args.steps):
        t.phase("merge", step.merge)
    torch.cuda.synchronize()
    check_device("in the standalone merge")
    m_ms = t.mean_ms("merge")
    gbs = step.merge_bytes / (m_ms / 1000.0) / 1e9
    return {"gbs": gbs, "ms": m_ms, "bytes": step.merge_bytes, "parts": len(step.o_parts),
            "frac_of_measured_hbm": gbs / peaks["hbm_gbs"], "in_timed_step": False,
            "roofline": hbm_roofline(step.merge_bytes, m_ms, peaks, "merge.ring_causal" if not args.seq_len else None)}


def latency_report(wname, dev, stream, peaks, reps=200):
    """A latency configuration: one sp_attn_fwd call (the config's head chunks and KV blocks) timed back to
    back through the C ABI (host enqueue included) and replayed from a CUDA graph (device only)."""
    import torch
    from sequence_head_attention_b200 import spattn, synth
    w = synth.WORKLOADS[wname]
    spattn.sp_set_launch_overlap(0)  # plain calls, each launch after the previous kernel
    q, k, v = (t.to(dev) for t in synth.qkv(w.B, w.S, w.H, w.D, seed=0, scale=w.scale)[:3])
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    ws_bytes = spattn.sp_attn_fwd_workspace_bytes(w.B, w.S, w.H, w.D, w.n_kv_blocks, False)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    chunks = list(w.head_chunks) if w.head_chunks else None

    def call():
        spattn.sp_attn_fwd(q, k, v, o, lse, head_chunks=chunks, n_kv_blocks=w.n_kv_blocks, workspace=ws)

    for _ in range(20):
        call()
    torch.cuda.synchronize(dev)
    check_device(f"in {wname}")
    t = Timer(stream)
    sampler = clock_sampler(dev).start()
    t.phase("calls", lambda: [call() for _ in range(reps)])
    torch.cuda.synchronize(dev)
    us_call = 1000.0 * t.mean_ms("calls") / reps
    flops = w.flops()
    launches = w.n_kv_blocks + (1 if w.n_kv_blocks > 1 else 0)
    rec = {"workload": workload_name(w, wname), "head_chunks": chunks, "kv_blocks": w.n_kv_blocks,
           "launches_per_call": launches, "flops_per_call": flops,
           "back_to_back": {"us_per_call": us_call, "tflops": flops / (us_call * 1e-6) / 1e12, "calls": reps}}
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            call()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g):
            for _ in range(10):
                call()
        g.replay()
        torch.cuda.synchronize(dev)
        t2 = Timer(stream)
        t2.phase("graph", lambda: [g.replay() for _ in range(reps // 10)])
        torch.cuda.synchronize(dev)
        check_device(f"in the {wname} graph replays")
        us_graph = 1000.0 * t2.mean_ms("graph") / (10 * (reps // 10))
        rec["cuda_graph"] = {"us_per_call": us_graph, "tflops": flops / (us_graph * 1e-6) / 1e12,
                             "calls": 10 * (reps // 10)}
        rec["roofline"] = tensor_roofline(flops, us_graph / 1000.0, peaks)
        del g
    except Exception as e:  # a capture problem is reported, not fatal
        rec["cuda_graph"] = {"error": f"{type(e).__name__}: {e}"[:200]}
        rec["roofline"] = tensor_roofline(flops, us_call / 1000.0, peaks)
    rec["roofline"]["note"] = "latency configuration: a handful of tiles, bound by launch latency, not by the tensor pipe"
    rec["clocks"] = sampler.stop()
    return rec


def e2e_report(wname, step, inp, args, dev, stream, world):
    """The same steps through the public API with host buffers: every step's inputs are copied from pinned
    host memory and its O read back into pinned host memory, inside the timed region.  A second step object
    gives the pipeline its second slot, so the copies of one step overlap the kernels of its neighbours."""
    import torch
    from sequence_head_attention_b200.pipeline import HostPipeline
    w, q, k, v, mask, fused = inp
    step2 = make_step(wname, w, q, k, v, mask, dev, fused)
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
    t = Timer(stream)
    t.phase("e2e", lambda: pipe.run(n_e2e, stream))
    torch.cuda.synchronize(dev)
    barrier()
    check_device("during the end-to-end steps")
    e_ms = max_over_ranks(t.mean_ms("e2e"), device=dev)
    return {"value": step.flops * n_e2e * world / (e_ms / 1000.0) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e, "ms_per_step": e_ms / n_e2e,
            "pipeline": "2 step slots; H2D, kernels and D2H on three streams, overlapped across steps"}


def free_gpu():
    import gc

    import torch
    gc.collect()
    torch.cuda.empty_cache()


def run_sp(args):
    """Real sequence parallelism over the N ranks (one GPU each): every rank holds only its sequence shard of
    the one global problem; Ulysses (video_dit) exchanges Q, K, V and O with NCCL all-to-alls, the ring
    (ring_causal) passes the KV blocks round the ranks with NCCL point-to-point sends, the library's kernels
    computing in between (sequence_head_attention_b200/dist.py).  Total work is fixed: strong scaling."""
    import torch
    from sequence_head_attention_b200 import dist as sp_dist
    from sequence_head_attention_b200 import spattn

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl", timeout_s=180, always=True)
    spattn.lib()
    stream = torch.cuda.current_stream(dev)
    peaks = measured_peaks()
    wname = "video_dit" if args.sp == "ulysses" else "ring_causal"
    w, q, k, v, _ = build_inputs(wname, seed=0)  # the same global problem on every rank
    Sl = w.S // world
    qs, ks, vs = (t[:, rank * Sl:(rank + 1) * Sl].contiguous().to(dev) for t in (q, k, v))
    del q, k, v
    if args.sp == "ulysses":
        sp = sp_dist.UlyssesAttention(w.B, w.S, w.H, w.D, head_chunks=w.head_chunks, causal=w.causal, device=dev,
                                      stages=args.sp_stages)
        flops_rank = w.flops() / world  # every rank attends H/P heads over the whole sequence
    else:
        sp = sp_dist.RingAttention(w.B, w.S, w.H, w.D, causal=w.causal, device=dev)
        # causal: rank r's queries see the blocks of ranks 0..r (its own one causally)
        blk = 4.0 * w.B * w.H * Sl * Sl * w.D
        flops_rank = blk * (rank + (0.5 if w.causal else 1.0)) if w.causal else blk * world
    o = torch.empty_like(qs)
    for _ in range(args.warmup):
        sp.forward(qs, ks, vs, out=o)
    torch.cuda.synchronize(dev)
    check_device("during the sequence-parallel warm-up")
    sampler = clock_sampler(dev).start()
    barrier()
    torch.cuda.synchronize(dev)
    timer = Timer(stream)
    t0, t1 = timer.E(), timer.E()
    t0.record(stream)
    for _ in range(args.steps):
        sp.forward(qs, ks, vs, out=o, phase=timer.phase)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    check_device("during the sequence-parallel steps")
    ms = max_over_ranks(t0.elapsed_time(t1), device=dev)
    value = w.flops() * args.steps / (ms / 1000.0) / 1e12
    attn_ms = sum(timer.spans("attn")) / args.steps  # this rank's attention launches per step
    exch = timer.spans("exchange")
    roofline = tensor_roofline(flops_rank, attn_ms, peaks)
    roofline["note"] = "this rank's attention launches of one step, timed together"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(config_of(w, wname, 1), parallelism=f"{args.sp}{world}",
                           global_batch=w.B, sp=f"{args.sp}: each rank holds S/{world} positions of Q, K, V",
                           sp_stages=args.sp_stages if args.sp == "ulysses" else None),
            "roofline": roofline, "cpu_baseline": None, "e2e": None,
            "gpu_launches": None, "clocks": clocks, "impl": "ours",
            "kernels": {"rank0": {"attention_ms_per_step": attn_ms, "flops_per_step": flops_rank,
                                  "exchange_ms_per_step": sum(exch) / args.steps if exch else 0.0,
                                  "bytes_sent_per_step": sp.bytes_exchanged(),
                                  "rounds": getattr(sp, "rounds", None)}}}
    emit(line, rank)
    del sp
    finish_dist()
    return 0


def run_ours(args):
    import torch
    from sequence_head_attention_b200 import spattn

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist("nccl", timeout_s=180)
    spattn.lib()  # fail now if the library is missing
    stream = torch.cuda.current_stream(dev)
    peaks = measured_peaks()
    head = "video_dit" if args.workload == "all" else args.workload
    if head in ("tiny_dense", "megatron"):
        raise SystemExit("--workload tiny_dense / megatron: latency configurations, measured under kernels "
                         "by the default run")

    rec, step, inp = measure_main(head, args, peaks, dev, stream, world, seed=rank, headline=True)
    w, q, k, v, mask, fused = inp
    kernels = {head: {key: rec[key] for key in rec if key not in ("clocks",)}}
    if head == "video_dit":
        if fused:
            kernels["relayout"] = relayout_report(step, args.steps, stream, peaks)
        if not args.no_backward:
            kernels["backward"] = backward_report(w, q, k, v, max(3, args.steps // 2), stream, peaks, dev)
    if head == "block_sparse" and args.dbsp_ranks > 1:
        kernels["dbsp"] = dbsp_ranks_report(step, args.dbsp_ranks, max(3, args.steps // 2), stream)
    roofline = rec["attention"]["roofline"]
    e2e = None if args.no_e2e else e2e_report(head, step, inp, args, dev, stream, world)
    launches = step.launches * args.steps
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = calibrated_oracle_baseline(head, q, k, v, mask, target_s=args.cpu_seconds)
    extra = {}
    if head == "video_dit":
        extra = {"ulysses": "attention on the sequence shards, relayouts folded into the kernel" if fused
                 else "seq->head relayout, per-rank attention, head->seq relayout"}
    if head == "block_sparse":
        extra = {"mask_density": step.density, "kept_tiles": step.kept_tiles}
    extra["launch_overlap"] = rec["launch_overlap"]
    line = {"metric": METRIC, "value": rec["tflops"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(w, head, world, extra), "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e, "gpu_launches": launches, "clocks": rec["clocks"], "impl": "ours"}
    del step, inp, q, k, v, mask
    free_gpu()

    if args.workload == "all":
        # every other configuration, each timed on its own (per rank when N > 1)
        for name in ("ring_causal", "block_sparse"):
            r2, s2, inp2 = measure_main(name, args, peaks, dev, stream, world, seed=rank, headline=False)
            if name == "block_sparse" and args.dbsp_ranks > 1:
                r2["dbsp"] = dbsp_ranks_report(s2, args.dbsp_ranks, max(3, args.steps // 2), stream)
            kernels[name] = r2
            del s2, inp2
            free_gpu()
        for name in ("tiny_dense", "megatron"):
            kernels[name] = latency_report(name, dev, stream, peaks)
            free_gpu()
    line["kernels"] = kernels
    line["config"]["other_configs"] = ("measured under kernels.<name>, each with its own CUDA-event timing and "
                                       "roofline" if args.workload == "all" else "not run (--workload)")
    emit(line, rank)
    finish_dist()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=("all",) + ALL_WORKLOADS, default="all",
                    help="all (default): the S=32K headline plus every other configuration under kernels; "
                         "a single full-size workload for profiling captures; tiny_dense / megatron: "
                         "reference arm only")
    ap.add_argument("--sp", choices=["replicas", "ulysses", "ring"], default="replicas",
                    help="replicas (default): every rank runs its own batch of every workload (weak scaling); "
                         "ulysses / ring: one global problem sequence-parallel over the ranks with NCCL "
                         "collectives (video_dit all-to-all, ring_causal ring; strong scaling)")
    ap.add_argument("--sp-stages", type=int, default=2,
                    help="--sp ulysses: head-chunk stages per rank (HCMS), each stage's all-to-all overlapping "
                         "the previous stage's attention")
    ap.add_argument("--ulysses", choices=["fused", "relayout"], default="fused",
                    help="video_dit step: attention straight on the sequence shards (fused), or the seq->head "
                         "relayout, per-rank attention and head->seq relayout")
    ap.add_argument("--dbsp-ranks", type=int, default=4,
                    help="block_sparse: also time the work split over this many simulated ranks, head split "
                         "vs db-SP plan (0: off)")
    ap.add_argument("--no-backward", action="store_true", help="video_dit: skip the backward-pass measurement")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch every attention kernel only after the previous kernel has completed")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=16, help="query rows per reference step")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override S of a single workload (profiling captures on a smaller case; not a "
                         "benchmark number)")
    ap.add_argument("--ranks", type=int, default=0,
                    help="override the simulated rank count of video_dit (profiling captures only)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if (args.seq_len or args.ranks) and args.workload == "all":
        ap.error("--seq-len / --ranks apply to a single --workload")
    if args.sp != "replicas":
        return run_sp(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
