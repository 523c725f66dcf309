"""Host-to-host pipeline over a stream of steps: each step's inputs arrive from pinned host memory and its
results go back to pinned host memory, and the copies of one step overlap the kernels of its neighbours.

A step object (workloads.UlyssesStep, RingStep, SparseStep) owns its device buffers, lists them with
``inputs()`` / ``outputs()`` and enqueues its kernels with ``run(stream)``.  The pipeline keeps ``depth`` such
objects (double buffering by default) and three CUDA streams:

    H2D stream      step i's inputs, host -> device, once step i - depth has finished computing on them;
    compute stream  step i's kernels, once its inputs have landed and step i - depth's results were read;
    D2H stream      step i's results, device -> host, once step i has computed them.

The copy engines move step i+1's inputs and step i-1's results while the SMs run step i, so a long stream of
steps runs at the pace of the slower of the copies and the kernels instead of their sum.  Nothing here
computes: it orders copies and launches with events.
"""
from __future__ import annotations

import torch


class HostPipeline:
    def __init__(self, steps, host_inputs, host_outputs):
        """steps: ``depth`` step objects of one workload (their buffers are the pipeline slots).
        host_inputs: pinned host tensors matching ``steps[0].inputs()``, the data every step reads.
        host_outputs: one list per slot of pinned host tensors matching ``steps[s].outputs()``."""
        if len(steps) < 1 or len(host_outputs) != len(steps):
            raise ValueError("one host output set per step slot")
        self.steps = steps
        self.h_in = host_inputs
        self.h_out = host_outputs
        dev = steps[0].inputs()[0].device
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)

    def run(self, n_steps: int, stream=None):
        """Enqueue n_steps steps; returns when everything is enqueued.  On return the given (or current)
        stream waits for the last result to reach the host, so an event recorded on it after this call
        marks the end of the whole run."""
        comp = stream or torch.cuda.current_stream(self.steps[0].inputs()[0].device)
        depth = len(self.steps)
        start = torch.cuda.Event()
        start.record(comp)
        self.h2d.wait_event(start)
        self.d2h.wait_event(start)
        in_ready = [torch.cuda.Event() for _ in range(depth)]
        computed = [torch.cuda.Event() for _ in range(depth)]
        read_back = [torch.cuda.Event() for _ in range(depth)]
        for i in range(n_steps):
            s = i % depth
            st = self.steps[s]
            if i >= depth:  # the slot's inputs are free once its previous step has computed
                self.h2d.wait_event(computed[s])
            with torch.cuda.stream(self.h2d):
                for h, t in zip(self.h_in, st.inputs()):
                    t.copy_(h, non_blocking=True)
                in_ready[s].record(self.h2d)
            comp.wait_event(in_ready[s])
            if i >= depth:  # ... and its outputs once they have been read back
                comp.wait_event(read_back[s])
            st.run(comp)
            computed[s].record(comp)
            self.d2h.wait_event(computed[s])
            with torch.cuda.stream(self.d2h):
                for h, t in zip(self.h_out[s], st.outputs()):
                    h.copy_(t, non_blocking=True)
                read_back[s].record(self.d2h)
        for s in range(min(depth, n_steps)):
            comp.wait_event(read_back[s])

    def bytes_per_step(self):
        h2d = sum(t.numel() * t.element_size() for t in self.steps[0].inputs())
        d2h = sum(t.numel() * t.element_size() for t in self.steps[0].outputs())
        return h2d, d2h
