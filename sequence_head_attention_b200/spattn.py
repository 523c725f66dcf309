"""ctypes binding of libspattn.so, one Python function per C entry point, same names.

Argument marshalling only: torch tensors supply device pointers and the stream; every step of the
computation runs in the library's CUDA kernels.  There is no fallback path: if the shared library is
missing or fails to load, every call raises.  The C contract (layouts, ownership, errors) is documented
in include/sp_attn.h.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspattn.so")
HEADER = os.path.join(_HERE, "..", "include", "sp_attn.h")

SP_OK, SP_ERR_INVALID_ARG, SP_ERR_UNSUPPORTED, SP_ERR_CUDA, SP_ERR_TIMEOUT = 0, 1, 2, 3, 4
SP_BF16, SP_F32 = 0, 1
SP_TILE = 128
SP_MAX_PARTS = 64
SP_MAX_RANKS = 64

_lock = threading.Lock()
_lib = None


class SpError(RuntimeError):
    """A libspattn call returned a status other than SP_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {sp_status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m sequence_head_attention_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_ulonglong
            sig = {
                "sp_attn_fwd_workspace_bytes": (Z, [I, I, I, I, I, I]),
                "sp_attn_fwd": (I, [P, P, P, P, P, I, I, I, I, P, I, I, I, P, P, Z, P]),
                "sp_attn_fwd_partial": (I, [P, P, P, P, P, I, I, I, I, I, I, I, P, P, Z, P]),
                "sp_attn_fwd_partial_merge": (I, [P, P, P, P, P, I, I, I, I, I, I, I, P, P, Z, P]),
                "sp_merge_partials": (I, [P, P, I, P, P, I, I, I, I, I, P]),
                "sp_seq_to_head_relayout": (I, [P, P, I, I, I, I, I, I, P]),
                "sp_head_to_seq_relayout": (I, [P, P, I, I, I, I, I, I, P]),
                "sp_attn_fwd_seq_sharded": (I, [P, P, P, P, P, I, I, I, I, I, I, I, P, I, I, P]),
                "sp_split_heads": (I, [P, P, I, I, I, I, I, I, I, I, P]),
                "sp_merge_heads": (I, [P, P, I, I, I, I, I, I, I, I, P]),
                "sp_attn_fwd_items": (I, [P, P, P, P, P, I, I, I, I, P, I, I, P, P, Z, P]),
                "sp_attn_bwd_workspace_bytes": (Z, [I, I, I, I]),
                "sp_attn_bwd": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, I, P, Z, P]),
                "sp_attn_bwd_partial": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, Z, P]),
                "sp_convert_f32_to_bf16": (I, [P, P, ctypes.c_longlong, P]),
                "sp_dbsp_unit_costs": (I, [P, I, I, I, P]),
                "sp_dbsp_plan": (I, [P, I, I, I, P, P, P]),
                "sp_dbsp_rank_items": (I, [P, P, I, I, I, I, P, I, P]),
                "sp_build_tile_list": (I, [P, I, I, P, P, P, P]),
                "sp_attn_fwd_sparse_noalloc": (I, [P, P, P, P, P, I, I, I, I, I, P, P]),
                "sp_status_string": (ctypes.c_char_p, [I]),
                "sp_check_device_error": (I, [P]),
                "sp_check_device_error_bits": (I, [P, P]),
                "sp_set_wait_timeout_ns": (None, [U64]),
                "sp_set_launch_overlap": (None, [I]),
                "sp_debug_wait_timeout": (I, [U64, P]),
                "sp_debug_exp2_poly": (I, [P, P, I, P]),
                "sp_version": (ctypes.c_char_p, []),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != SP_OK:
        raise SpError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def _need(cond, msg):
    if not cond:
        raise ValueError(msg)


def _bshd(t, name, dtype=torch.bfloat16):
    _need(t.dim() == 4, f"{name} must be [B, S, H, D]")
    _need(t.dtype == dtype, f"{name} must be {dtype}")
    _need(t.is_cuda and t.is_contiguous(), f"{name} must be a contiguous CUDA tensor")


def _same_device(ts, ref):
    for t in ts:
        if t is not None:
            _need(t.device == ref.device, "all tensors must be on one device")


def _check_mask(block_mask, H, S, device):
    """A block mask the kernels may read: contiguous uint8 [H, ceil(S/128), ceil(S/128)] on `device`.  The
    library receives only a pointer, so a wrong shape or a host tensor is refused here, before any call."""
    T = (S + SP_TILE - 1) // SP_TILE
    _need(isinstance(block_mask, torch.Tensor) and block_mask.dtype == torch.uint8 and block_mask.is_contiguous(),
          "block_mask must be a contiguous uint8 tensor")
    _need(tuple(block_mask.shape) == (H, T, T), f"block_mask must be [H, ceil(S/128), ceil(S/128)] = [{H}, {T}, {T}]")
    _need(block_mask.is_cuda and block_mask.device == torch.device(device),
          "block_mask must be a CUDA tensor on the device of q")


def _check_lse(lse, B, H, S, device):
    """An lse output the kernels may write: contiguous fp32 [B, H, S] on `device`."""
    _need(isinstance(lse, torch.Tensor) and lse.dtype == torch.float32 and lse.is_contiguous()
          and tuple(lse.shape) == (B, H, S), "lse must be contiguous fp32 [B, H, S]")
    _need(lse.is_cuda and lse.device == torch.device(device), "lse must be a CUDA tensor on the device of q")


# ------------------------------------------------------------------------------------------------------
def sp_status_string(status: int) -> str:
    return lib().sp_status_string(int(status)).decode()


def sp_version() -> str:
    return lib().sp_version().decode()


def sp_attn_fwd_workspace_bytes(B, S, H, D, n_kv_blocks=1, has_mask=False) -> int:
    return int(lib().sp_attn_fwd_workspace_bytes(B, S, H, D, n_kv_blocks, int(bool(has_mask))))


def sp_attn_fwd(q, k, v, o, lse=None, head_chunks=None, n_kv_blocks=1, causal=False, block_mask=None,
                workspace=None, stream=None):
    """Exact attention of q, k, v (bf16 [B,S,H,D]) into o (bf16) and lse (fp32 [B,H,S] or None).

    The workspace, when the configuration needs one and none is given, is allocated here with torch
    (device memory is the caller's: the library itself never allocates)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bshd(t, n)
    _same_device((k, v, o), q)
    B, S, H, D = q.shape
    if lse is not None:
        _check_lse(lse, B, H, S, q.device)
    if block_mask is not None:
        _check_mask(block_mask, H, S, q.device)
    ws_bytes = sp_attn_fwd_workspace_bytes(B, S, H, D, n_kv_blocks, block_mask is not None)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    hc = None
    n_hc = 0
    if head_chunks is not None:
        n_hc = len(head_chunks)
        hc = (ctypes.c_int * n_hc)(*[int(c) for c in head_chunks])
    st = lib().sp_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S, H, D,
                           ctypes.cast(hc, ctypes.c_void_p) if hc is not None else None, n_hc,
                           int(n_kv_blocks), int(bool(causal)), _ptr(block_mask), _ptr(workspace),
                           0 if workspace is None else workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check("sp_attn_fwd", st)
    return o, lse


def sp_attn_fwd_partial(q, k, v, o_part, lse_part, kv_begin, kv_end, causal=False, block_mask=None,
                        workspace=None, stream=None):
    """One KV block [kv_begin, kv_end) for every query: fp32 o_part [B,S,H,D], fp32 lse_part [B,H,S]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bshd(t, n)
    _bshd(o_part, "o_part", torch.float32)
    _same_device((k, v, o_part), q)
    B, S, H, D = q.shape
    _need(tuple(o_part.shape) == (B, S, H, D), "o_part must be [B, S, H, D]")
    _check_lse(lse_part, B, H, S, q.device)
    if block_mask is not None:
        _check_mask(block_mask, H, S, q.device)
    ws_bytes = sp_attn_fwd_workspace_bytes(B, S, H, D, 1, block_mask is not None)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    st = lib().sp_attn_fwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, S, H, D,
                                   int(kv_begin), int(kv_end), int(bool(causal)), _ptr(block_mask),
                                   _ptr(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check("sp_attn_fwd_partial", st)
    return o_part, lse_part


def sp_attn_fwd_partial_merge(q, k, v, o_acc, lse_acc, kv_begin, kv_end, causal=False, block_mask=None,
                              workspace=None, stream=None):
    """One KV block [kv_begin, kv_end) merged in place into the running result o_acc (fp32 [B,S,H,D]) and
    lse_acc (fp32 [B,H,S]); rows that see no key of the block are left untouched."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _bshd(t, n)
    _bshd(o_acc, "o_acc", torch.float32)
    _same_device((k, v, o_acc), q)
    B, S, H, D = q.shape
    _need(tuple(o_acc.shape) == (B, S, H, D), "o_acc must be [B, S, H, D]")
    _check_lse(lse_acc, B, H, S, q.device)
    if block_mask is not None:
        _check_mask(block_mask, H, S, q.device)
    ws_bytes = sp_attn_fwd_workspace_bytes(B, S, H, D, 1, block_mask is not None)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    st = lib().sp_attn_fwd_partial_merge(_ptr(q), _ptr(k), _ptr(v), _ptr(o_acc), _ptr(lse_acc), B, S, H, D,
                                         int(kv_begin), int(kv_end), int(bool(causal)), _ptr(block_mask),
                                         _ptr(workspace),
                                         0 if workspace is None else workspace.numel() * workspace.element_size(),
                                         _stream(stream))
    _check("sp_attn_fwd_partial_merge", st)
    return o_acc, lse_acc


def sp_merge_partials(o_parts, lse_parts, o, lse=None, stream=None):
    """Log-sum-exp re-merge of n fp32 partials into o (bf16 or fp32 [B,S,H,D]) and lse (fp32 [B,H,S])."""
    n = len(o_parts)
    _need(n == len(lse_parts) and n >= 1, "need n >= 1 matching partials")
    B, S, H, D = o_parts[0].shape
    dt = SP_F32 if o.dtype == torch.float32 else SP_BF16
    _need(o.dtype in (torch.float32, torch.bfloat16), "o must be fp32 or bf16")
    for t in o_parts:
        _need(t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (B, S, H, D), "bad o_part")
    for t in lse_parts:
        _need(t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (B, H, S), "bad lse_part")
    op, _keep1 = _ptr_array(o_parts)
    lp, _keep2 = _ptr_array(lse_parts)
    st = lib().sp_merge_partials(op, lp, n, _ptr(o), _ptr(lse), dt, B, S, H, D, _stream(stream))
    _check("sp_merge_partials", st)
    return o, lse


def sp_seq_to_head_relayout(in_ranks, out_ranks, S=None, H=None, stream=None):
    """P rank buffers [B, S/P, H, D] -> P rank buffers [B, S, H/P, D] (bit-exact)."""
    P = len(in_ranks)
    B, Sl, H_, D = in_ranks[0].shape
    S = Sl * P if S is None else S
    H = H_ if H is None else H
    ip, _k1 = _ptr_array(in_ranks)
    op, _k2 = _ptr_array(out_ranks)
    st = lib().sp_seq_to_head_relayout(ip, op, P, B, S, H, D, in_ranks[0].element_size(), _stream(stream))
    _check("sp_seq_to_head_relayout", st)
    return out_ranks


def sp_head_to_seq_relayout(in_ranks, out_ranks, S=None, H=None, stream=None):
    """P rank buffers [B, S, H/P, D] -> P rank buffers [B, S/P, H, D] (bit-exact)."""
    P = len(in_ranks)
    B, S_, Hl, D = in_ranks[0].shape
    S = S_ if S is None else S
    H = Hl * P if H is None else H
    ip, _k1 = _ptr_array(in_ranks)
    op, _k2 = _ptr_array(out_ranks)
    st = lib().sp_head_to_seq_relayout(ip, op, P, B, S, H, D, in_ranks[0].element_size(), _stream(stream))
    _check("sp_head_to_seq_relayout", st)
    return out_ranks


def sp_split_heads(x, out_ranks, heads=None, stream=None):
    """x [B, S, H, D] (this rank's sequence shard) -> P head groups out_ranks[r] [B, S, n, D] holding heads
    [r H/P + h0, r H/P + h0 + n) with heads=(h0, n) (default: each whole group), bit-exact."""
    P = len(out_ranks)
    B, S, H, D = x.shape
    h0, n = (0, H // P) if heads is None else (int(heads[0]), int(heads[1]))
    _need(x.is_cuda and x.is_contiguous(), "x must be a contiguous CUDA tensor")
    for t in out_ranks:
        _need(t.is_cuda and t.is_contiguous() and t.dtype == x.dtype and tuple(t.shape) == (B, S, n, D)
              and t.device == x.device, "out_ranks must be contiguous [B, S, n, D] of x's dtype and device")
    op, _k = _ptr_array(out_ranks)
    _check("sp_split_heads", lib().sp_split_heads(_ptr(x), op, P, B, S, H, D, h0, n, x.element_size(),
                                                  _stream(stream)))
    return out_ranks


def sp_merge_heads(in_ranks, out, heads=None, stream=None):
    """P head groups in_ranks[r] [B, S, n, D] -> heads [r H/P + h0, r H/P + h0 + n) of out [B, S, H, D] with
    heads=(h0, n) (default: each whole group), bit-exact; out's other heads are left untouched."""
    P = len(in_ranks)
    B, S, H, D = out.shape
    h0, n = (0, H // P) if heads is None else (int(heads[0]), int(heads[1]))
    _need(out.is_cuda and out.is_contiguous(), "out must be a contiguous CUDA tensor")
    for t in in_ranks:
        _need(t.is_cuda and t.is_contiguous() and t.dtype == out.dtype and tuple(t.shape) == (B, S, n, D)
              and t.device == out.device, "in_ranks must be contiguous [B, S, n, D] of out's dtype and device")
    ip, _k = _ptr_array(in_ranks)
    _check("sp_merge_heads", lib().sp_merge_heads(ip, _ptr(out), P, B, S, H, D, h0, n, out.element_size(),
                                                  _stream(stream)))
    return out


def sp_attn_fwd_seq_sharded(q_shards, k_shards, v_shards, o_shards, lse=None, heads=None, head_chunks=None,
                            causal=False, stream=None):
    """One Ulysses rank's attention on the sequence shards (bf16 [B, S/P, H, D] each, P of them):
    heads [h0, h0 + n) with heads=(h0, n) (default: all), written into the heads of o_shards; lse is
    fp32 [B, H, S] over all heads (rows of the computed heads written) or None.  Bit-identical to the
    seq -> head relayout, sp_attn_fwd on those heads, and the head -> seq relayout."""
    P = len(q_shards)
    _need(P >= 1 and len(k_shards) == P and len(v_shards) == P and len(o_shards) == P, "P shards of each")
    for group, n in ((q_shards, "q"), (k_shards, "k"), (v_shards, "v"), (o_shards, "o")):
        for i, t in enumerate(group):
            _bshd(t, f"{n}_shards[{i}]")
            _need(t.shape == q_shards[0].shape, "all shards must have the same shape")
    B, Sl, H, D = q_shards[0].shape
    S = Sl * P
    h0, n = (0, H) if heads is None else (int(heads[0]), int(heads[1]))
    if lse is not None:
        _need(lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, H, S),
              "lse must be contiguous fp32 [B, H, S]")
    hc = None
    n_hc = 0
    if head_chunks is not None:
        n_hc = len(head_chunks)
        hc = (ctypes.c_int * n_hc)(*[int(c) for c in head_chunks])
    qp, _k1 = _ptr_array(q_shards)
    kp, _k2 = _ptr_array(k_shards)
    vp, _k3 = _ptr_array(v_shards)
    op, _k4 = _ptr_array(o_shards)
    st = lib().sp_attn_fwd_seq_sharded(qp, kp, vp, op, _ptr(lse), P, B, S, H, D, h0, n,
                                       ctypes.cast(hc, ctypes.c_void_p) if hc is not None else None, n_hc,
                                       int(bool(causal)), _stream(stream))
    _check("sp_attn_fwd_seq_sharded", st)
    return o_shards, lse


def sp_dbsp_unit_costs(block_mask, H, T, causal=False):
    """Host: kept tiles per (head, query-tile pair) unit, int64 [H, ceil(T/2)] (block_mask: host uint8
    [H, T, T] tensor or array, or None for dense)."""
    import numpy as np
    NP = (T + 1) // 2
    cost = np.zeros((H, NP), dtype=np.int64)
    m = None
    if block_mask is not None:
        m = np.ascontiguousarray(block_mask.cpu().numpy() if isinstance(block_mask, torch.Tensor) else block_mask,
                                 dtype=np.uint8)
        _need(m.shape == (H, T, T), "block_mask must be [H, T, T]")
    st = lib().sp_dbsp_unit_costs(None if m is None else m.ctypes.data, H, T, int(bool(causal)), cost.ctypes.data)
    _check("sp_dbsp_unit_costs", st)
    return cost


def sp_dbsp_plan(cost, P):
    """Host: (unit_rank int32 [H, NP], rank_load int64 [P], imbalance) of the two-level partition."""
    import numpy as np
    cost = np.ascontiguousarray(cost, dtype=np.int64)
    H, NP = cost.shape
    unit_rank = np.zeros((H, NP), dtype=np.int32)
    load = np.zeros(P, dtype=np.int64)
    imb = ctypes.c_double(0.0)
    st = lib().sp_dbsp_plan(cost.ctypes.data, H, NP, int(P), unit_rank.ctypes.data, load.ctypes.data,
                            ctypes.byref(imb))
    _check("sp_dbsp_plan", st)
    return unit_rank, load, imb.value


def sp_dbsp_rank_items(cost, unit_rank, B, rank):
    """Host: int32 kernel item ids of one rank, longest unit first."""
    import numpy as np
    cost = np.ascontiguousarray(cost, dtype=np.int64)
    unit_rank = np.ascontiguousarray(unit_rank, dtype=np.int32)
    H, NP = cost.shape
    n = ctypes.c_int(0)
    _check("sp_dbsp_rank_items", lib().sp_dbsp_rank_items(cost.ctypes.data, unit_rank.ctypes.data, B, H, NP,
                                                          int(rank), None, 0, ctypes.byref(n)))
    items = np.zeros(max(n.value, 1), dtype=np.int32)
    _check("sp_dbsp_rank_items", lib().sp_dbsp_rank_items(cost.ctypes.data, unit_rank.ctypes.data, B, H, NP,
                                                          int(rank), items.ctypes.data, n.value, ctypes.byref(n)))
    return items[:n.value]


def sp_attn_fwd_items(q, k, v, o, lse, items, causal=False, block_mask=None, workspace=None, stream=None):
    """Attention of the listed work items only (items: device int32 tensor of item ids)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bshd(t, n)
    _same_device((k, v, o, items), q)
    B, S, H, D = q.shape
    _need(items.dtype == torch.int32 and items.is_cuda and items.is_contiguous(), "items must be CUDA int32")
    if lse is not None:
        _check_lse(lse, B, H, S, q.device)
    if block_mask is not None:
        _check_mask(block_mask, H, S, q.device)
    ws_bytes = sp_attn_fwd_workspace_bytes(B, S, H, D, 1, block_mask is not None)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    st = lib().sp_attn_fwd_items(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S, H, D, _ptr(items),
                                 items.numel(), int(bool(causal)), _ptr(block_mask), _ptr(workspace),
                                 0 if workspace is None else workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check("sp_attn_fwd_items", st)
    return o, lse


def sp_attn_bwd(q, k, v, o, dout, lse, dq, dk, dv, causal=False, workspace=None, stream=None):
    """Gradients dq, dk, dv (bf16 [B,S,H,D]) of the attention for the upstream gradient dout, from the
    forward's o and lse.  The fp32 delta workspace is allocated here with torch when none is given."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _bshd(t, n)
    B, S, H, D = q.shape
    _need(lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, H, S),
          "lse must be contiguous fp32 [B, H, S]")
    ws_bytes = lib().sp_attn_bwd_workspace_bytes(B, S, H, D)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    st = lib().sp_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                           _ptr(dv), B, S, H, D, int(bool(causal)), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check("sp_attn_bwd", st)
    return dq, dk, dv


def sp_attn_bwd_partial(q, k, v, o, dout, lse, dq_acc, dk, dv, kv_begin, kv_end, causal=False, workspace=None,
                        stream=None):
    """Backward of one KV block [kv_begin, kv_end) (o, lse: the merged forward result): writes dk, dv rows
    of the block and adds its dq contribution into dq_acc (fp32 [B,S,H,D])."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout"), (dk, "dk"), (dv, "dv")):
        _bshd(t, n)
    _bshd(dq_acc, "dq_acc", torch.float32)
    B, S, H, D = q.shape
    _need(lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, H, S),
          "lse must be contiguous fp32 [B, H, S]")
    ws_bytes = lib().sp_attn_bwd_workspace_bytes(B, S, H, D)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    st = lib().sp_attn_bwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq_acc), _ptr(dk),
                                   _ptr(dv), B, S, H, D, int(kv_begin), int(kv_end), int(bool(causal)),
                                   _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("sp_attn_bwd_partial", st)
    return dq_acc, dk, dv


def sp_convert_f32_to_bf16(x, out, stream=None):
    """out (bf16) = x (fp32) rounded to nearest even; same number of elements, a multiple of 4."""
    _need(x.dtype == torch.float32 and out.dtype == torch.bfloat16 and x.numel() == out.numel(), "f32 in, bf16 out")
    _need(x.is_contiguous() and out.is_contiguous(), "contiguous tensors")
    _check("sp_convert_f32_to_bf16", lib().sp_convert_f32_to_bf16(_ptr(x), _ptr(out), x.numel(), _stream(stream)))
    return out


def sp_attn_fwd_sparse_noalloc(q, k, v, o, lse, block_mask, causal=False, stream=None):
    """Block-sparse attention with no workspace: for callers that cannot allocate device memory.

    Same result as sp_attn_fwd(..., block_mask=block_mask); the mask's tile list goes into a fixed
    array inside the library instead (size limits and the no-overlap rule in include/sp_attn.h)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bshd(t, n)
    _same_device((k, v, o), q)
    B, S, H, D = q.shape
    _need(block_mask is not None, "block_mask is required")
    _check_mask(block_mask, H, S, q.device)
    if lse is not None:
        _check_lse(lse, B, H, S, q.device)
    st = lib().sp_attn_fwd_sparse_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S, H, D,
                                          int(bool(causal)), _ptr(block_mask), _stream(stream))
    _check("sp_attn_fwd_sparse_noalloc", st)
    return o, lse


def sp_build_tile_list(block_mask, S, row_ptr, col_idx, counts, stream=None):
    """CSR of the kept key tiles of a uint8 [H, T, T] block mask (T = ceil(S/128))."""
    H = block_mask.shape[0]
    _check_mask(block_mask, H, S, block_mask.device)
    T = (S + SP_TILE - 1) // SP_TILE
    for t, n, size in ((row_ptr, "row_ptr", H * T + 1), (col_idx, "col_idx", H * T * T), (counts, "counts", H * T)):
        _need(t.dtype == torch.int32 and t.is_contiguous() and t.numel() >= size and t.device == block_mask.device,
              f"{n} must be a contiguous int32 tensor of at least {size} elements on the mask's device")
    st = lib().sp_build_tile_list(_ptr(block_mask), H, S, _ptr(row_ptr), _ptr(col_idx), _ptr(counts),
                                  _stream(stream))
    _check("sp_build_tile_list", st)
    return row_ptr, col_idx


def sp_check_device_error(stream=None) -> int:
    """Synchronise the stream; return SP_ERR_TIMEOUT if a bounded device wait expired since the last check."""
    return int(lib().sp_check_device_error(_stream(stream)))


def sp_check_device_error_bits(stream=None):
    """(status, bits): the raw device error word, one bit per kind of wait that expired."""
    bits = ctypes.c_uint(0)
    st = lib().sp_check_device_error_bits(_stream(stream), ctypes.byref(bits))
    return int(st), int(bits.value)


def sp_set_wait_timeout_ns(ns: int) -> None:
    lib().sp_set_wait_timeout_ns(int(ns))


def sp_set_launch_overlap(mode) -> None:
    """Let each attention launch start while the kernel before it on the stream finishes: 0 (or False) off,
    1 (or True) early reads of q, k, v only, 2 also outputs written without waiting (see the header for
    what the caller promises in each mode)."""
    lib().sp_set_launch_overlap(int(mode))


def sp_debug_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check("sp_debug_wait_timeout", lib().sp_debug_wait_timeout(int(timeout_ns), _stream(stream)))


def sp_debug_exp2_poly(x, y, stream=None):
    """The kernels' FMA-pipe 2^x on a CUDA fp32 tensor x (even length) into y."""
    _need(x.dtype == torch.float32 and y.dtype == torch.float32 and x.numel() % 2 == 0, "fp32, even length")
    _check("sp_debug_exp2_poly", lib().sp_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def declared_symbols():
    """The entry points include/sp_attn.h declares (parsed from the header)."""
    import re
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:[\w\*\s]+?)\b(sp_\w+)\s*\(", text, re.M)))
