"""fp64 CPU oracle for the sequence/head-parallel attention path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs may import
this package.  It shares no code with ``sequence_head_attention_b200`` and never imports it.

The arithmetic lives in ``sp_oracle.c`` (plain C, double precision); this module compiles it with gcc
on first use and marshals numpy arrays.  Each function's docstring names the passage it follows; the C
file's header carries the full list.

Every function here is pinned by ``tests/test_oracle_pins.py`` to properties the pages or plain
mathematics fix (brute force, closed forms, invariants, a library routine); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sp_oracle.c")
_LIB = os.path.join(_HERE, "libsporacle.so")
_lock = threading.Lock()
_libs = {}

TILE = 128


def compile_source(src: str, out: str) -> str:
    """Compile one oracle C source into a shared library (gcc, -O2, no fast-math, no FMA contraction)."""
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared",
           "-pthread", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``sp_oracle.c`` into ``libsporacle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _load(path: str | None = None):
    with _lock:
        key = path or _LIB
        if key not in _libs:
            lib = ctypes.CDLL(path or build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.orc_attn.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, I, I, P, I, I]
            lib.orc_attn_probs.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, I, I, I]
            lib.orc_merge.argtypes = [P, P, I, P, P, I, I, I, I]
            lib.orc_seq_to_head.argtypes = [P, P, I, I, I, I, I, I]
            lib.orc_head_to_seq.argtypes = [P, P, I, I, I, I, I, I]
            lib.orc_split_heads.argtypes = [P, P, I, I, I, I, I, I]
            lib.orc_merge_heads.argtypes = [P, P, I, I, I, I, I, I]
            lib.orc_tile_list.argtypes = [P, I, I, I, P, P, ctypes.c_long]
            lib.orc_attn_bwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I]
            for f in (lib.orc_attn, lib.orc_attn_probs, lib.orc_merge, lib.orc_seq_to_head,
                      lib.orc_head_to_seq, lib.orc_split_heads, lib.orc_merge_heads, lib.orc_tile_list,
                      lib.orc_attn_bwd):
                f.restype = ctypes.c_int
            _libs[key] = lib
    return _libs[key]


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _mask_arg(block_mask, H, S, tile):
    if block_mask is None:
        return None
    m = np.ascontiguousarray(np.asarray(block_mask, dtype=np.uint8))
    nt = (S + tile - 1) // tile
    if m.shape != (H, nt, nt):
        raise ValueError(f"block_mask must be [H, {nt}, {nt}], got {m.shape}")
    return m


def attention(q, k, v, *, causal=False, block_mask=None, tile=TILE, kv_begin=0, kv_end=None,
              rows=None, nthreads=None, lib=None):
    """Exact attention per head, in fp64, from its definition (two-pass softmax).

    Follows "LLM Lab Notes 05: Attention Tensor Parallelism", section 2 step 4 and its explanation
    (per head: q @ k^T / sqrt(head_dim), softmax over keys, weighted sum of v), with the key set
    narrowed by causality, by a KV range (one Ring-Attention round, "CHARM+: How Cross-Hardware
    Attention Breaks Through ...", Ring-Attention paragraph) and by a per-head block mask ("db-SP",
    abstract).

    q, k, v: [B, S, H, D].  rows: optional query positions; then o is [B, len(rows), H, D] and lse is
    [B, H, len(rows)].  Returns (o, lse) in fp64; lse is the natural-log log-sum-exp of the scaled
    scores, -inf for a row without keys (whose o is 0).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one [B, S, H, D] shape")
    kv_end = S if kv_end is None else kv_end
    m = _mask_arg(block_mask, H, S, tile)
    rows_a = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    n_out = S if rows_a is None else len(rows_a)
    o = np.zeros((B, n_out, H, D))
    lse = np.zeros((B, H, n_out))
    nthreads = nthreads or os.cpu_count() or 1
    rc = _load(lib).orc_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S, H, D, int(causal),
                          _ptr(m), tile, kv_begin, kv_end, _ptr(rows_a),
                          0 if rows_a is None else len(rows_a), nthreads)
    if rc:
        raise ValueError(f"orc_attn failed ({rc})")
    return o, lse


def attention_bwd(q, k, v, dout, *, causal=False, nthreads=None, lib=None):
    """Gradients (dq, dk, dv) of the exact attention, in fp64, for an upstream gradient dout of o.

    The backward pass whose speed "CHARM+ ..." (abstract) reports, written as plain calculus on the same
    definition as :func:`attention` (all keys, optionally causal): dv_j = sum_i p_ij do_i;
    dp_ij = do_i . v_j; delta_i = sum_j p_ij dp_ij; ds_ij = p_ij (dp_ij - delta_i);
    dq_i = sum_j ds_ij k_j / sqrt(D); dk_j = sum_i ds_ij q_i / sqrt(D).  All arrays [B, S, H, D]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, S, H, D = q.shape
    for t in (k, v, dout):
        if t.shape != q.shape:
            raise ValueError("q, k, v, dout must share one [B, S, H, D] shape")
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    nthreads = nthreads or os.cpu_count() or 1
    rc = _load(lib).orc_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, S, H,
                              D, int(causal), nthreads)
    if rc:
        raise ValueError(f"orc_attn_bwd failed ({rc})")
    return dq, dk, dv


def attention_bwd_rows(q, k, v, dout, *, heads, q_rows, k_rows, causal=False, nthreads=None, lib=None):
    """dq at the query positions q_rows and dk, dv at the key positions k_rows, for the listed heads, in
    fp64: the same definitions as :func:`attention_bwd` ("CHARM+ ...", abstract: the backward pass),
    evaluated one row at a time.  The forward o and lse of every query of those heads come from
    :func:`attention`; then, with p_ij = exp(q_i.k_j / sqrt(D) - lse_i) and delta_i = do_i . o_i,
    dq_i = sum_j p_ij (do_i.v_j - delta_i) k_j / sqrt(D) over the keys query i sees, and
    dv_j = sum_i p_ij do_i, dk_j = sum_i p_ij (do_i.v_j - delta_i) q_i / sqrt(D) over the queries that
    see key j.  A row costs O(S D), so full-size workloads can be checked on sampled rows.

    Returns dq [B, len(q_rows), len(heads), D] and dk, dv [B, len(k_rows), len(heads), D]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, S, H, D = q.shape
    hs = [int(h) for h in heads]
    qh, kh, vh, dh = (np.ascontiguousarray(t[:, :, hs]) for t in (q, k, v, dout))
    o, lse = attention(qh, kh, vh, causal=causal, nthreads=nthreads, lib=lib)
    delta = np.einsum("bshd,bshd->bhs", dh, o)
    scale = 1.0 / np.sqrt(D)
    dq = np.zeros((B, len(q_rows), len(hs), D))
    dk = np.zeros((B, len(k_rows), len(hs), D))
    dv = np.zeros((B, len(k_rows), len(hs), D))
    for b in range(B):
        for n_h in range(len(hs)):
            Q, K, V, dO = qh[b, :, n_h], kh[b, :, n_h], vh[b, :, n_h], dh[b, :, n_h]
            L, dl = lse[b, n_h], delta[b, n_h]
            for n, i in enumerate(q_rows):
                je = i + 1 if causal else S  # keys query i sees
                p = np.exp(K[:je] @ Q[i] * scale - L[i])
                ds = p * (V[:je] @ dO[i] - dl[i])
                dq[b, n, n_h] = ds @ K[:je] * scale
            for n, j in enumerate(k_rows):
                i0 = j if causal else 0  # queries that see key j
                p = np.exp(Q[i0:] @ K[j] * scale - L[i0:])
                dv[b, n, n_h] = p @ dO[i0:]
                ds = p * (dO[i0:] @ V[j] - dl[i0:])
                dk[b, n, n_h] = ds @ Q[i0:] * scale
    return dq, dk, dv


def attention_probs(q, k, v, *, causal=False, block_mask=None, tile=TILE, kv_begin=0, kv_end=None, lib=None):
    """As :func:`attention`, also returning the probabilities p [B, H, S, S] (tiny inputs only)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, H, D = q.shape
    kv_end = S if kv_end is None else kv_end
    m = _mask_arg(block_mask, H, S, tile)
    o = np.zeros((B, S, H, D))
    lse = np.zeros((B, H, S))
    p = np.zeros((B, H, S, S))
    rc = _load(lib).orc_attn_probs(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(p), B, S, H, D,
                                int(causal), _ptr(m), tile, kv_begin, kv_end)
    if rc:
        raise ValueError(f"orc_attn_probs failed ({rc})")
    return o, lse, p


def merge(o_parts, lse_parts, *, lib=None):
    """Re-merge KV-block partials with the log-sum-exp rule ("CHARM+: Cross-Hardware Attention with
    Re-Merge Multistream Mechanism", abstract: re-merge of partial results).

    o_parts: n arrays [B, S, H, D]; lse_parts: n arrays [B, H, S].  Returns (o, lse) in fp64.
    """
    os_ = [_f64(a) for a in o_parts]
    ls_ = [_f64(a) for a in lse_parts]
    n = len(os_)
    if n < 1 or len(ls_) != n:
        raise ValueError("need n >= 1 matching partials")
    B, S, H, D = os_[0].shape
    o = np.zeros((B, S, H, D))
    lse = np.zeros((B, H, S))
    op = (ctypes.c_void_p * n)(*[a.ctypes.data for a in os_])
    lp = (ctypes.c_void_p * n)(*[a.ctypes.data for a in ls_])
    rc = _load(lib).orc_merge(ctypes.cast(op, ctypes.c_void_p), ctypes.cast(lp, ctypes.c_void_p), n,
                           _ptr(o), _ptr(lse), B, S, H, D)
    if rc:
        raise ValueError(f"orc_merge failed ({rc})")
    return o, lse


def _relayout(fn, in_ranks, out_shape, P):
    ins = [np.ascontiguousarray(a) for a in in_ranks]
    if len(ins) != P:
        raise ValueError("need P input buffers")
    dt = ins[0].dtype
    outs = [np.zeros(out_shape, dtype=dt) for _ in range(P)]
    ip = (ctypes.c_void_p * P)(*[a.ctypes.data for a in ins])
    op = (ctypes.c_void_p * P)(*[a.ctypes.data for a in outs])
    return ins, outs, ip, op


def seq_to_head(in_ranks, H, *, lib=None):
    """Ulysses seq-shard -> head-shard permutation ("HCMS", abstract; "db-SP", abstract).

    in_ranks: P arrays [B, S/P, H, D] (any dtype).  Returns P arrays [B, S, H/P, D]:
    out_r[b, s, h'] = in_{s // (S/P)}[b, s % (S/P), r*H/P + h'].
    """
    P = len(in_ranks)
    B, Sl, H_, D = np.asarray(in_ranks[0]).shape
    if H_ != H or H % P:
        raise ValueError("bad head count")
    S = Sl * P
    ins, outs, ip, op = _relayout(None, in_ranks, (B, S, H // P, D), P)
    rc = _load(lib).orc_seq_to_head(ctypes.cast(ip, ctypes.c_void_p), ctypes.cast(op, ctypes.c_void_p),
                                 P, B, S, H, D, ins[0].itemsize)
    if rc:
        raise ValueError(f"orc_seq_to_head failed ({rc})")
    return outs


def head_to_seq(in_ranks, S, *, lib=None):
    """Inverse of :func:`seq_to_head`: P arrays [B, S, H/P, D] -> P arrays [B, S/P, H, D]."""
    P = len(in_ranks)
    B, S_, Hl, D = np.asarray(in_ranks[0]).shape
    if S_ != S or S % P:
        raise ValueError("bad sequence length")
    H = Hl * P
    ins, outs, ip, op = _relayout(None, in_ranks, (B, S // P, H, D), P)
    rc = _load(lib).orc_head_to_seq(ctypes.cast(ip, ctypes.c_void_p), ctypes.cast(op, ctypes.c_void_p),
                                 P, B, S, H, D, ins[0].itemsize)
    if rc:
        raise ValueError(f"orc_head_to_seq failed ({rc})")
    return outs


def split_heads(x, P, *, lib=None):
    """One rank's half of the Ulysses all-to-all on the way in ("HCMS", abstract: all-to-all sequence
    parallelism, here between processes): its sequence shard x [B, S, H, D] cut into P head groups,
    out_r [B, S, H/P, D] = x[:, :, r*H/P : (r+1)*H/P] (the block it sends to rank r)."""
    xa = np.ascontiguousarray(x)
    B, S, H, D = xa.shape
    if H % P:
        raise ValueError("bad head count")
    outs = [np.zeros((B, S, H // P, D), dtype=xa.dtype) for _ in range(P)]
    op = (ctypes.c_void_p * P)(*[a.ctypes.data for a in outs])
    rc = _load(lib).orc_split_heads(xa.ctypes.data_as(ctypes.c_void_p), ctypes.cast(op, ctypes.c_void_p), P, B, S,
                                    H, D, xa.itemsize)
    if rc:
        raise ValueError(f"orc_split_heads failed ({rc})")
    return outs


def merge_heads(parts, *, lib=None):
    """The way back: P head groups [B, S, H/P, D] (group r from rank r) joined into [B, S, H, D]."""
    ins = [np.ascontiguousarray(a) for a in parts]
    P = len(ins)
    B, S, Hl, D = ins[0].shape
    out = np.zeros((B, S, Hl * P, D), dtype=ins[0].dtype)
    ip = (ctypes.c_void_p * P)(*[a.ctypes.data for a in ins])
    rc = _load(lib).orc_merge_heads(ctypes.cast(ip, ctypes.c_void_p), out.ctypes.data_as(ctypes.c_void_p), P, B, S,
                                    Hl * P, D, ins[0].itemsize)
    if rc:
        raise ValueError(f"orc_merge_heads failed ({rc})")
    return out


def tile_list(block_mask, *, lib=None):
    """CSR of kept key tiles per (head, query tile): (row_ptr [H*Tq+1] int32, col_idx [nnz] int32)."""
    m = np.ascontiguousarray(np.asarray(block_mask, dtype=np.uint8))
    H, Tq, Tk = m.shape
    cap = int(np.count_nonzero(m))
    row_ptr = np.zeros(H * Tq + 1, dtype=np.int32)
    col_idx = np.zeros(max(cap, 1), dtype=np.int32)
    rc = _load(lib).orc_tile_list(_ptr(m), H, Tq, Tk, _ptr(row_ptr), _ptr(col_idx), cap)
    if rc:
        raise ValueError(f"orc_tile_list failed ({rc})")
    return row_ptr, col_idx[:cap]
