"""The host-to-host pipeline (two step slots, copies on their own streams) returns, for every step, the
same O as running the step on its own with its inputs already on the device."""
import pytest
import torch

from sequence_head_attention_b200 import spattn, synth, workloads
from sequence_head_attention_b200.pipeline import HostPipeline

pytestmark = pytest.mark.gpu


def _pinned_like(ts):
    return [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ts]


@pytest.mark.parametrize("kind", ["ulysses_fused", "ulysses_relayout", "ring", "sparse"])
def test_pipeline_matches_direct_run(kind):
    if kind.startswith("ulysses"):
        w = synth.Workload("small_ulysses", 1, 1000, 8, 128, 0.5, False, (3, 5), 1, 4)
    elif kind == "ring":
        w = synth.Workload("small_ring", 1, 1024, 4, 128, 0.5, True, (4,), 4, 1)
    else:
        w = synth.Workload("small_sparse", 1, 1024, 4, 64, 0.5, False, (4,), 1, 1, True)
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=11, scale=w.scale)
    mask = synth.block_mask(w.H, w.S, seed=11) if w.sparse else None

    def make():
        if kind.startswith("ulysses"):
            return workloads.UlyssesStep(w, q, k, v, fused=kind == "ulysses_fused")
        if kind == "ring":
            return workloads.RingStep(w, q, k, v)
        return workloads.SparseStep(w, q, k, v, mask)

    ref = make()
    ref.run()
    torch.cuda.synchronize()
    expect = [t.cpu() for t in ref.outputs()]

    slots = [make(), make()]
    for s in slots:  # garbage in the device buffers: every step must bring its own inputs
        for t in s.inputs():
            t.fill_(7.0)
    h_in = _pinned_like(ref.inputs())
    for h, t in zip(h_in, ref.inputs()):
        h.copy_(t)
    h_out = [_pinned_like(s.outputs()) for s in slots]
    pipe = HostPipeline(slots, h_in, h_out)
    for n in (1, 3):
        for hs in h_out:
            for h in hs:
                h.fill_(-1.0)
        pipe.run(n)
        torch.cuda.synchronize()
        assert spattn.sp_check_device_error() == spattn.SP_OK
        for s in range(min(n, 2)):
            for h, e in zip(h_out[s], expect):
                assert torch.equal(h, e)
