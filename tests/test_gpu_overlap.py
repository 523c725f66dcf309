"""Launch overlap (sp_set_launch_overlap): attention launches that start while the kernel before them on the
stream finishes must write exactly what they write without overlap.  Checked on the launch sequences the
benchmark overlaps: per-rank launches on sequence shards (disjoint heads of shared output buffers), the
ring's merging launches (each reads the previous one's running result), and masked launches (their tile
list is built by the kernels just before), each repeated so that launches really follow one another."""
import pytest
import torch

from sequence_head_attention_b200 import spattn, synth
from sequence_head_attention_b200.synth import Workload
from sequence_head_attention_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture
def overlap():
    spattn.sp_set_launch_overlap(1)
    yield
    spattn.sp_set_launch_overlap(0)


def _run(fn, mode):
    spattn.sp_set_launch_overlap(mode)
    out = fn()
    torch.cuda.synchronize()
    st, bits = spattn.sp_check_device_error_bits()
    assert st == spattn.SP_OK, hex(bits)
    return [t.clone() for t in out]


def test_rank_launches_on_shards(overlap):
    w = Workload("shards", 1, 8192, 16, 128, 0.5, False, (3, 5, 8), 1, 4)
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=7, scale=0.5)
    step = workloads.UlyssesStep(w, q, k, v, fused=True)

    def go():
        for _ in range(3):
            step.run()
        return step.o_seq + [step.lse_all]

    ref = _run(go, 0)
    for mode in (1, 2):  # mode 2: the ranks write disjoint heads, so outputs are written without waiting
        got = _run(go, mode)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_ring_merging_launches(overlap):
    w = Workload("ring", 1, 8192, 8, 128, 0.5, True, (8,), 8, 1)
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=8, scale=0.5)
    step = workloads.RingStep(w, q, k, v)

    def go():
        for _ in range(3):
            step.run()
        return [step.o, step.lse]

    ref = _run(go, 0)
    got = _run(go, 1)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_masked_launches(overlap):
    w = Workload("sparse", 1, 4096, 8, 128, 0.5, False, (8,), 1, 1, True)
    q, k, v = synth.qkv(w.B, w.S, w.H, w.D, seed=9, scale=0.5)
    step = workloads.SparseStep(w, q, k, v, synth.block_mask(w.H, w.S, seed=9))

    def go():
        for _ in range(3):
            step.run()
        return [step.o, step.lse]

    ref = _run(go, 0)
    got = _run(go, 1)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
