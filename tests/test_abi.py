"""The C-ABI library builds, loads without a GPU, exports every entry point include/sp_attn.h declares,
and rejects invalid arguments on the host before any launch (no compute call is made here)."""
import ctypes
import subprocess

import pytest

from sequence_head_attention_b200 import build as sp_build
from sequence_head_attention_b200 import spattn


@pytest.fixture(scope="module")
def L():
    sp_build.build()
    return spattn.lib()


def test_every_declared_symbol_is_exported(L):
    declared = spattn.declared_symbols()
    assert len(declared) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", spattn.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert getattr(L, s) is not None


def test_status_strings_and_version(L):
    assert spattn.sp_status_string(0) == "SP_OK"
    assert spattn.sp_status_string(4) == "SP_ERR_TIMEOUT"
    assert "sm_100a" in spattn.sp_version()


def test_workspace_bytes_arithmetic(L):
    assert spattn.sp_attn_fwd_workspace_bytes(1, 256, 4, 64, 1, False) == 0
    # two fp32 partials of O [1,256,4,64] and LSE [1,4,256], each rounded up to 256 bytes
    assert spattn.sp_attn_fwd_workspace_bytes(1, 256, 4, 64, 2, False) == 2 * 256 * 4 * 64 * 4 + 2 * 4 * 256 * 4
    T = 2
    mask_bytes = (256 * (-(-(4 * T + 1) * 4 // 256)) + 256 * (-(-(4 * T * T) * 4 // 256)) + 256 * (-(-(4 * T) * 4 // 256))
                  + 256 * (-(-(1 * 4 * ((T + 1) // 2)) * 4 // 256)))  # row_ptr, col_idx, counts, work order
    assert spattn.sp_attn_fwd_workspace_bytes(1, 256, 4, 64, 1, True) == mask_bytes
    assert spattn.sp_attn_fwd_workspace_bytes(1, 256, 4, 96, 1, False) == 0  # D must be 64 or 128


def _attn(L, q=16, k=16, v=16, o=16, B=1, S=256, H=4, D=64, chunks=None, n_kv=1, causal=0):
    hc = None if chunks is None else (ctypes.c_int * len(chunks))(*chunks)
    return L.sp_attn_fwd(q, k, v, o, None, B, S, H, D, ctypes.cast(hc, ctypes.c_void_p) if hc else None,
                         0 if chunks is None else len(chunks), n_kv, causal, None, None, 0, None)


@pytest.mark.parametrize("kw", [
    dict(D=96), dict(D=0), dict(B=0), dict(S=0), dict(H=0),
    dict(q=0), dict(o=0), dict(q=24),                       # null / misaligned pointers
    dict(chunks=[1, 2]), dict(chunks=[2, 2, 1]), dict(chunks=[0, 4]), dict(chunks=[-1, 5]),
    dict(n_kv=0), dict(n_kv=3), dict(causal=2),            # n_kv_blocks > ceil(S/128) = 2
    dict(n_kv=2),                                          # needs a workspace, none given
])
def test_attn_fwd_rejects_on_host(L, kw):
    assert _attn(L, **kw) == spattn.SP_ERR_INVALID_ARG


def test_partial_and_merge_reject_on_host(L):
    st = L.sp_attn_fwd_partial(16, 16, 16, 16, 16, 1, 256, 4, 64, 10, 5, 0, None, None, 0, None)
    assert st == spattn.SP_ERR_INVALID_ARG  # kv_end < kv_begin
    st = L.sp_attn_fwd_partial(16, 16, 16, 16, 16, 1, 256, 4, 64, 0, 300, 0, None, None, 0, None)
    assert st == spattn.SP_ERR_INVALID_ARG  # kv_end > S
    st = L.sp_attn_fwd_partial(16, 16, 16, 16, 16, 1, 256, 4, 64, 64, 256, 0, 16, None, 0, None)
    assert st == spattn.SP_ERR_INVALID_ARG  # masked block must start on a tile boundary
    arr = (ctypes.c_void_p * 2)(16, 32)
    p = ctypes.cast(arr, ctypes.c_void_p)
    assert L.sp_merge_partials(p, p, 0, 64, None, 0, 1, 8, 1, 64, None) == spattn.SP_ERR_INVALID_ARG
    assert L.sp_merge_partials(p, p, 65, 64, None, 0, 1, 8, 1, 64, None) == spattn.SP_ERR_INVALID_ARG
    assert L.sp_merge_partials(p, p, 2, 64, None, 7, 1, 8, 1, 64, None) == spattn.SP_ERR_INVALID_ARG
    assert L.sp_merge_partials(p, p, 2, 16, None, 0, 1, 8, 1, 64, None) == spattn.SP_ERR_INVALID_ARG  # bf16 in place


def test_relayout_rejects_on_host(L):
    ins = (ctypes.c_void_p * 4)(1 << 20, 2 << 20, 3 << 20, 4 << 20)
    outs = (ctypes.c_void_p * 4)(5 << 20, 6 << 20, 7 << 20, 8 << 20)
    i, o = ctypes.cast(ins, ctypes.c_void_p), ctypes.cast(outs, ctypes.c_void_p)
    f = L.sp_seq_to_head_relayout
    assert f(i, o, 4, 1, 30, 8, 64, 2, None) == spattn.SP_ERR_INVALID_ARG   # S % P
    assert f(i, o, 4, 1, 32, 6, 64, 2, None) == spattn.SP_ERR_INVALID_ARG   # H % P
    assert f(i, o, 4, 1, 32, 8, 4, 2, None) == spattn.SP_ERR_INVALID_ARG    # D * elem not a multiple of 16
    assert f(i, o, 4, 1, 32, 8, 64, 3, None) == spattn.SP_ERR_INVALID_ARG   # elem_bytes
    assert f(i, o, 0, 1, 32, 8, 64, 2, None) == spattn.SP_ERR_INVALID_ARG   # P
    assert f(i, o, 65, 1, 65, 65, 64, 2, None) == spattn.SP_ERR_INVALID_ARG  # P > SP_MAX_RANKS
    overlap = (ctypes.c_void_p * 4)(1 << 20, 6 << 20, 7 << 20, 8 << 20)     # out 0 aliases in 0
    assert f(i, ctypes.cast(overlap, ctypes.c_void_p), 4, 1, 32, 8, 64, 2, None) == spattn.SP_ERR_INVALID_ARG
    assert L.sp_head_to_seq_relayout(i, o, 4, 1, 30, 8, 64, 2, None) == spattn.SP_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(spattn, "_lib", None)
    monkeypatch.setattr(spattn, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        spattn.sp_version()


def test_binding_refuses_bad_masks_and_lse_before_any_call():
    """The library gets only pointers, so the binding refuses a mask or lse of the wrong shape, type or
    device before calling it (a host or undersized mask would be read out of bounds by the kernels)."""
    import torch
    S, H = 1000, 3  # T = ceil(1000 / 128) = 8
    good = torch.zeros((H, 8, 8), dtype=torch.uint8)
    with pytest.raises(ValueError, match=r"\[3, 8, 8\]"):
        spattn._check_mask(torch.zeros((H, 7, 8), dtype=torch.uint8), H, S, "cuda:0")
    with pytest.raises(ValueError, match=r"\[3, 8, 8\]"):
        spattn._check_mask(torch.zeros((H + 1, 8, 8), dtype=torch.uint8), H, S, "cuda:0")
    with pytest.raises(ValueError, match="uint8"):
        spattn._check_mask(good.float(), H, S, "cuda:0")
    with pytest.raises(ValueError, match="uint8"):
        spattn._check_mask(torch.zeros((H, 8, 16), dtype=torch.uint8)[:, :, ::2], H, S, "cuda:0")
    with pytest.raises(ValueError, match="CUDA"):
        spattn._check_mask(good, H, S, "cuda:0")  # a host tensor
    with pytest.raises(ValueError, match="lse"):
        spattn._check_lse(torch.zeros((1, H, S - 1)), 1, H, S, "cuda:0")
    with pytest.raises(ValueError, match="lse"):
        spattn._check_lse(torch.zeros((1, H, S), dtype=torch.float64), 1, H, S, "cuda:0")
    with pytest.raises(ValueError, match="CUDA"):
        spattn._check_lse(torch.zeros((1, H, S)), 1, H, S, "cuda:0")
    # the tile-list wrapper checks its mask too, before touching the library
    i32 = torch.zeros(H * 64, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        spattn.sp_build_tile_list(good, S, i32, i32, i32)


def test_partial_merge_rejects_on_host(L):
    f = L.sp_attn_fwd_partial_merge
    q, o, l = 1 << 24, 2 << 24, 3 << 24  # distinct, 16-byte aligned, never dereferenced
    assert f(q, q, q, o, None, 1, 256, 4, 64, 0, 128, 0, None, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, o, l, 1, 256, 4, 64, 10, 5, 0, None, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, o, l, 1, 256, 4, 64, 0, 300, 0, None, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, o, l, 1, 256, 4, 64, 64, 256, 0, 16, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, q + 64, l, 1, 256, 4, 64, 0, 256, 0, None, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, o, o + 64, 1, 256, 4, 64, 0, 256, 0, None, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, o, l, 1, 256, 4, 96, 0, 256, 0, None, None, 0, None) == spattn.SP_ERR_INVALID_ARG
    assert f(q, q, q, o, l, 1, 256, 4, 64, 128, 128, 0, None, None, 0, None) == spattn.SP_OK  # empty: no launch


def test_split_and_merge_heads_reject_on_host(L):
    outs = (ctypes.c_void_p * 4)(1 << 24, 2 << 24, 3 << 24, 4 << 24)
    o = ctypes.cast(outs, ctypes.c_void_p)
    x = 5 << 24
    f, g = L.sp_split_heads, L.sp_merge_heads
    assert f(x, o, 4, 1, 16, 6, 64, 0, 1, 2, None) == spattn.SP_ERR_INVALID_ARG     # H % P
    assert f(x, o, 4, 1, 16, 8, 4, 0, 2, 2, None) == spattn.SP_ERR_INVALID_ARG      # D * elem not a multiple of 16
    assert f(x, o, 4, 1, 16, 8, 64, 0, 2, 3, None) == spattn.SP_ERR_INVALID_ARG     # elem_bytes
    assert f(x + 8, o, 4, 1, 16, 8, 64, 0, 2, 2, None) == spattn.SP_ERR_INVALID_ARG  # misaligned
    assert f(x, o, 4, 1, 16, 8, 64, 1, 2, 2, None) == spattn.SP_ERR_INVALID_ARG     # heads past the group (2)
    assert f(x, o, 4, 1, 16, 8, 64, 0, 0, 2, None) == spattn.SP_ERR_INVALID_ARG     # no head
    assert f(1 << 24, o, 4, 1, 16, 8, 64, 0, 2, 2, None) == spattn.SP_ERR_INVALID_ARG  # input overlaps output 0
    same = (ctypes.c_void_p * 4)(1 << 24, 1 << 24, 3 << 24, 4 << 24)
    assert f(x, ctypes.cast(same, ctypes.c_void_p), 4, 1, 16, 8, 64, 0, 2, 2, None) == spattn.SP_ERR_INVALID_ARG
    assert g(o, x, 0, 1, 16, 8, 64, 0, 2, 2, None) == spattn.SP_ERR_INVALID_ARG     # P
    assert g(o, 2 << 24, 4, 1, 16, 8, 64, 0, 2, 2, None) == spattn.SP_ERR_INVALID_ARG  # output overlaps input 1
