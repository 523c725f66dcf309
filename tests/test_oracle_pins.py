"""Pins for the fp64 oracle: each test checks it against something other than itself.

What the pages fix: the per-head definition of attention ("LLM Lab Notes 05", section 2 step 4), the
equivalence of head-chunked and full attention and the rank-ordered concatenation check (same page,
sections 4 and 5; "HCMS", abstract: numerical equivalence under uneven head partitions), the traversal
of every KV block with accumulated partials (CHARM+ article, Ring-Attention paragraph) and the printed
output shape (tests/golden/p4_output_shape.json).  What mathematics fixes: brute-force evaluation on
tiny inputs, a library routine (torch SDPA in float64), closed forms (constant V, zero Q, single key),
invariants (permutation, self-merge, merge order) and index formulas written independently.

The last block plants mistakes in a copy of the oracle's C source and checks that the pins catch them.
"""
import json
import math
import os
import re
import tempfile

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(12345)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def brute_force(q, k, v, allowed):
    """Direct exp(s)/sum(exp(s)) without any max shift: valid for the small magnitudes used here.

    allowed(b, h, i, j) -> bool.  Returns (o, lse) with lse = ln sum exp(s)."""
    B, S, H, D = q.shape
    o = np.zeros_like(q)
    lse = np.full((B, H, S), -np.inf)
    for b in range(B):
        for h in range(H):
            for i in range(S):
                num = np.zeros(D)
                den = 0.0
                for j in range(S):
                    if not allowed(b, h, i, j):
                        continue
                    w = math.exp(float(np.dot(q[b, i, h], k[b, j, h])) / math.sqrt(D))
                    num += w * v[b, j, h]
                    den += w
                if den > 0:
                    o[b, i, h] = num / den
                    lse[b, h, i] = math.log(den)
    return o, lse


def assert_lse_equal(a, b, tol):
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    fin = np.isfinite(b)
    assert np.all(np.isfinite(a[fin]))
    if fin.any():
        assert np.max(np.abs(a[fin] - b[fin])) < tol


# ---------------------------------------------------------------------------------------------------
# Attention against brute force and a library routine
# ---------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_attention_brute_force_dense(causal):
    q, k, v = rand(2, 9, 3, 5), rand(2, 9, 3, 5), rand(2, 9, 3, 5)
    o, lse = oracle.attention(q, k, v, causal=causal)
    ob, lb = brute_force(q, k, v, lambda b, h, i, j: (not causal) or j <= i)
    assert np.max(np.abs(o - ob)) < 1e-12
    assert_lse_equal(lse, lb, 1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_torch_sdpa_fp64(causal):
    """Dense and causal attention reduce to a library routine: torch SDPA in float64 on the CPU."""
    B, S, H, D = 2, 37, 3, 16
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    o, _ = oracle.attention(q, k, v, causal=causal)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    ref = ref.permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(o - ref)) < 1e-12


def test_attention_brute_force_mask_and_kv_range():
    B, S, H, D, T = 1, 11, 2, 4, 3
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    nt = (S + T - 1) // T
    mask = (RNG.random((H, nt, nt)) < 0.5).astype(np.uint8)
    mask[:, 0, :] = 0  # query tile 0 sees nothing: empty rows
    kb, ke = 2, 9
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal=causal, block_mask=mask, tile=T, kv_begin=kb, kv_end=ke)
        allowed = lambda b, h, i, j: (kb <= j < ke and mask[h, i // T, j // T] != 0
                                      and ((not causal) or j <= i))
        ob, lb = brute_force(q, k, v, allowed)
        assert np.max(np.abs(o - ob)) < 1e-12
        assert_lse_equal(lse, lb, 1e-12)
        assert np.all(o[:, :T] == 0) and np.all(np.isneginf(lse[:, :, :T]))


def test_rows_subset_equals_full_rows():
    q, k, v = rand(2, 20, 2, 8), rand(2, 20, 2, 8), rand(2, 20, 2, 8)
    rows = [0, 3, 19, 7]
    of, lf = oracle.attention(q, k, v, causal=True)
    os_, ls = oracle.attention(q, k, v, causal=True, rows=rows)
    assert np.array_equal(os_, of[:, rows])
    assert np.array_equal(ls, lf[:, :, rows])


def test_thread_count_does_not_change_results():
    q, k, v = rand(1, 64, 3, 8), rand(1, 64, 3, 8), rand(1, 64, 3, 8)
    a = oracle.attention(q, k, v, nthreads=1)
    b = oracle.attention(q, k, v, nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------------------------------------------
# Closed forms and invariants
# ---------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    B, S, H, D, T = 1, 13, 2, 6, 4
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    nt = (S + T - 1) // T
    mask = (RNG.random((H, nt, nt)) < 0.6).astype(np.uint8)
    mask[:, np.arange(nt), np.arange(nt)] = 1
    _, lse, p = oracle.attention_probs(q, k, v, causal=causal, block_mask=mask, tile=T)
    sums = p.sum(axis=-1)
    assert np.max(np.abs(sums - 1.0)) < 1e-12
    assert np.all(p >= 0)
    for h in range(H):
        for i in range(S):
            for j in range(S):
                if (causal and j > i) or not mask[h, i // T, j // T]:
                    assert p[0, h, i, j] == 0.0


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_returns_v(causal):
    B, S, H, D = 2, 17, 3, 8
    q, k = rand(B, S, H, D, scale=2.0), rand(B, S, H, D, scale=2.0)
    c = rand(1, 1, H, D)
    v = np.broadcast_to(c, (B, S, H, D)).copy()
    o, _ = oracle.attention(q, k, v, causal=causal)
    assert np.max(np.abs(o - np.broadcast_to(c, o.shape))) < 1e-12


def test_zero_q_gives_uniform_weights():
    """q = 0 makes every score 0: o is the mean of v over the allowed keys and lse = ln |J|."""
    B, S, H, D, T = 1, 21, 2, 4, 5
    q = np.zeros((B, S, H, D))
    k, v = rand(B, S, H, D), rand(B, S, H, D)
    nt = (S + T - 1) // T
    mask = (RNG.random((H, nt, nt)) < 0.5).astype(np.uint8)
    mask[:, np.arange(nt), np.arange(nt)] = 1
    kb, ke = 3, 19
    for causal, m, (a, e) in [(False, None, (0, S)), (True, None, (0, S)), (False, mask, (0, S)),
                              (True, mask, (kb, ke))]:
        o, lse = oracle.attention(q, k, v, causal=causal, block_mask=m, tile=T, kv_begin=a, kv_end=e)
        for h in range(H):
            for i in range(S):
                J = [j for j in range(a, min(e, S)) if (not causal or j <= i)
                     and (m is None or m[h, i // T, j // T])]
                if not J:
                    assert np.all(o[0, i, h] == 0) and lse[0, h, i] == -np.inf
                    continue
                assert np.max(np.abs(o[0, i, h] - v[0, J, h].mean(axis=0))) < 1e-12
                assert abs(lse[0, h, i] - math.log(len(J))) < 1e-12


def test_single_key():
    """|J| = 1: o = v_0 and lse = q.k_0 / sqrt(D) (S = 1, and causal row 0)."""
    D = 32
    q, k, v = rand(1, 1, 2, D), rand(1, 1, 2, D), rand(1, 1, 2, D)
    o, lse = oracle.attention(q, k, v)
    assert np.max(np.abs(o - v)) < 1e-12
    for h in range(2):
        assert abs(lse[0, h, 0] - np.dot(q[0, 0, h], k[0, 0, h]) / math.sqrt(D)) < 1e-12
    q, k, v = rand(1, 9, 2, D), rand(1, 9, 2, D), rand(1, 9, 2, D)
    o, lse = oracle.attention(q, k, v, causal=True)
    assert np.max(np.abs(o[0, 0] - v[0, 0])) < 1e-12
    for h in range(2):
        assert abs(lse[0, h, 0] - np.dot(q[0, 0, h], k[0, 0, h]) / math.sqrt(D)) < 1e-12


def test_closed_form_three_keys():
    """D = 1, q = 1, k = (0, ln 2, ln 3): weights (1, 2, 3)/6.  v = (6, 0, 2) gives o = 2, lse = ln 6;
    causal rows give (6, 0), (2, ln 3), (2, ln 6)."""
    q = np.ones((1, 3, 1, 1))
    k = np.array([0.0, math.log(2), math.log(3)]).reshape(1, 3, 1, 1)
    v = np.array([6.0, 0.0, 2.0]).reshape(1, 3, 1, 1)
    o, lse = oracle.attention(q, k, v)
    assert np.allclose(o[0, :, 0, 0], [2, 2, 2], atol=1e-14, rtol=0)
    assert np.allclose(lse[0, 0], [math.log(6)] * 3, atol=1e-14, rtol=0)
    o, lse = oracle.attention(q, k, v, causal=True)
    assert np.allclose(o[0, :, 0, 0], [6, 2, 2], atol=1e-14, rtol=0)
    assert np.allclose(lse[0, 0], [0, math.log(3), math.log(6)], atol=1e-14, rtol=0)


def test_key_permutation_invariance():
    q, k, v = rand(1, 30, 2, 8), rand(1, 30, 2, 8), rand(1, 30, 2, 8)
    perm = RNG.permutation(30)
    a = oracle.attention(q, k, v)
    b = oracle.attention(q, k[:, perm], v[:, perm])
    assert np.max(np.abs(a[0] - b[0])) < 1e-12
    assert np.max(np.abs(a[1] - b[1])) < 1e-12


def test_all_ones_mask_equals_dense_and_diagonal_mask_is_per_tile():
    B, S, H, D, T = 1, 22, 2, 4, 5  # ragged last tile (22 = 4*5 + 2)
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    nt = (S + T - 1) // T
    ones = np.ones((H, nt, nt), dtype=np.uint8)
    for causal in (False, True):
        a = oracle.attention(q, k, v, causal=causal)
        b = oracle.attention(q, k, v, causal=causal, block_mask=ones, tile=T)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    diag = np.zeros((H, nt, nt), dtype=np.uint8)
    diag[:, np.arange(nt), np.arange(nt)] = 1
    o, lse = oracle.attention(q, k, v, block_mask=diag, tile=T)
    for t in range(nt):
        sl = slice(t * T, min(S, (t + 1) * T))
        ot, lt = oracle.attention(q[:, sl], k[:, sl], v[:, sl])
        assert np.max(np.abs(o[:, sl] - ot)) < 1e-12
        assert np.max(np.abs(lse[:, :, sl] - lt)) < 1e-12


def test_scale_of_inputs_stays_finite():
    q, k, v = rand(1, 256, 2, 128), rand(1, 256, 2, 128), rand(1, 256, 2, 128)
    for s in (0.5, 1.0, 8.0):
        o, lse = oracle.attention(q * s, k, v, causal=True)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))


# ---------------------------------------------------------------------------------------------------
# Head chunks (HCMS / Megatron head split)
# ---------------------------------------------------------------------------------------------------
def test_head_chunks_equal_full_and_wrong_order_fails():
    """Per-rank outputs of 8 heads each, concatenated in rank order along the hidden dimension, equal
    full attention ("LLM Lab Notes 05", sections 4-5); a permuted concatenation must not."""
    with open(os.path.join(GOLDEN, "p4_output_shape.json")) as f:
        g = json.load(f)
    cfg = g["config"]
    B, S, H = cfg["batch"], 16, cfg["heads"]  # full seq 128 is covered by the GPU tests
    D = cfg["hidden"] // H
    world = cfg["world"]
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    full, full_lse = oracle.attention(q, k, v)
    per = H // world
    outs, lses = [], []
    for r in range(world):
        hs = slice(r * per, (r + 1) * per)
        o_r, l_r = oracle.attention(q[:, :, hs], k[:, :, hs], v[:, :, hs])
        outs.append(o_r.reshape(B, S, per * D))
        lses.append(l_r)
    cat = np.concatenate(outs, axis=-1)
    assert np.array_equal(cat, full.reshape(B, S, H * D))  # bitwise: per-head math is unchanged
    assert np.array_equal(np.concatenate(lses, axis=1), full_lse)
    wrong = np.concatenate(outs[1:] + outs[:1], axis=-1)
    assert wrong.shape == cat.shape and not np.allclose(wrong, cat)


def test_uneven_head_chunks_equal_full():
    B, S, H, D = 1, 24, 40, 8
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    full, _ = oracle.attention(q, k, v)
    h0 = 0
    parts = []
    for c in (3, 7, 10, 10, 10):
        o_c, _ = oracle.attention(q[:, :, h0:h0 + c], k[:, :, h0:h0 + c], v[:, :, h0:h0 + c])
        parts.append(o_c)
        h0 += c
    assert np.array_equal(np.concatenate(parts, axis=2), full)


def test_printed_output_shape():
    """The page prints torch.Size([4, 128, 4096]) for batch 4, seq 128, hidden 4096, 32 heads."""
    with open(os.path.join(GOLDEN, "p4_output_shape.json")) as f:
        g = json.load(f)
    cfg = g["config"]
    B, S, H = cfg["batch"], cfg["seq"], cfg["heads"]
    D = cfg["hidden"] // H
    q = rand(B, S, H, D, scale=0.1)
    o, _ = oracle.attention(q, q, q, rows=[0, S - 1])
    assert list(o.shape[:1]) + [S, H * D] == g["output_shape"]
    assert (B, S, H * D) == tuple(g["output_shape"])


# ---------------------------------------------------------------------------------------------------
# KV blocks and the re-merge
# ---------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bounds", [(0, 16, 32), (0, 5, 11, 32), (0, 4, 8, 12, 16, 20, 24, 28, 32)])
def test_kv_block_partials_merge_to_full(causal, bounds):
    B, S, H, D = 2, 32, 2, 8
    q, k, v = rand(B, S, H, D), rand(B, S, H, D), rand(B, S, H, D)
    full = oracle.attention(q, k, v, causal=causal)
    parts = [oracle.attention(q, k, v, causal=causal, kv_begin=a, kv_end=e)
             for a, e in zip(bounds[:-1], bounds[1:])]
    o, lse = oracle.merge([p[0] for p in parts], [p[1] for p in parts])
    assert np.max(np.abs(o - full[0])) < 1e-12
    assert np.max(np.abs(lse - full[1])) < 1e-12


def test_merge_identities():
    B, S, H, D = 1, 12, 2, 4
    o1, l1 = rand(B, S, H, D), rand(B, H, S)
    o2, l2 = rand(B, S, H, D), rand(B, H, S)
    o3, l3 = rand(B, S, H, D), rand(B, H, S)
    l2[0, 1, 3] = -np.inf
    m = oracle.merge([o1], [l1])
    assert np.array_equal(m[0], o1) and np.array_equal(m[1], l1)
    m = oracle.merge([o1, o1], [l1, l1])
    assert np.max(np.abs(m[0] - o1)) < 1e-12
    assert np.max(np.abs(m[1] - (l1 + math.log(2)))) < 1e-12
    a = oracle.merge([o1, o2, o3], [l1, l2, l3])
    b = oracle.merge([o3, o1, o2], [l3, l1, l2])
    assert np.max(np.abs(a[0] - b[0])) < 1e-12 and np.max(np.abs(a[1] - b[1])) < 1e-12
    # two parts with weights: lse = ln(e^a + e^b), o = (e^a o1 + e^b o2) / (e^a + e^b)
    c = oracle.merge([o1, o2], [l1, l2])
    ea, eb = np.exp(l1), np.exp(l2)
    ref_l = np.log(ea + eb)
    wa = np.transpose(ea / (ea + eb), (0, 2, 1))[..., None]
    wb = np.transpose(eb / (ea + eb), (0, 2, 1))[..., None]
    assert np.max(np.abs(c[1] - ref_l)) < 1e-12
    assert np.max(np.abs(c[0] - (wa * o1 + wb * o2))) < 1e-12
    # all parts empty: o = 0, lse = -inf, never NaN
    e = np.full((B, H, S), -np.inf)
    z = oracle.merge([o1, o2], [e, e])
    assert np.all(z[0] == 0) and np.all(np.isneginf(z[1]))


# ---------------------------------------------------------------------------------------------------
# Relayout and tile list
# ---------------------------------------------------------------------------------------------------
@pytest.mark.parametrize("P,B,S,H,D", [(4, 1, 24, 8, 6), (2, 2, 10, 6, 3), (1, 2, 6, 3, 4), (3, 1, 9, 9, 2)])
def test_relayout_index_formula_and_round_trip(P, B, S, H, D):
    full = RNG.integers(0, 2**16, size=(B, S, H, D), dtype=np.uint16)
    shards = [full[:, r * (S // P):(r + 1) * (S // P)].copy() for r in range(P)]
    outs = oracle.seq_to_head(shards, H)
    for r in range(P):  # rank r owns heads [r*H/P, (r+1)*H/P) over the whole sequence
        assert np.array_equal(outs[r], full[:, :, r * (H // P):(r + 1) * (H // P)])
    back = oracle.head_to_seq(outs, S)
    for r in range(P):
        assert np.array_equal(back[r], shards[r])
    if P == 1:
        assert np.array_equal(outs[0], shards[0])


def test_relayout_byte_exact_for_float_payloads():
    P, B, S, H, D = 2, 1, 8, 4, 5
    full = rand(B, S, H, D).astype(np.float32)
    full[0, 1, 2, 3] = np.nan
    shards = [full[:, r * 4:(r + 1) * 4].copy() for r in range(P)]
    outs = oracle.seq_to_head(shards, H)
    assert outs[0].tobytes() == full[:, :, :2].copy().tobytes()
    assert outs[1].tobytes() == full[:, :, 2:].copy().tobytes()


@pytest.mark.parametrize("P,B,S,H,D", [(4, 1, 6, 8, 6), (2, 2, 5, 6, 3), (1, 2, 3, 3, 4), (3, 1, 4, 9, 2)])
def test_split_and_merge_heads_against_slices_and_the_exchange(P, B, S, H, D):
    """The local halves of a multi-process Ulysses exchange: split_heads equals numpy slicing of the head
    axis, merge_heads inverts it, and split on every rank followed by the all-to-all block transpose
    (rank r receives block r of every rank, in rank order along the sequence) is the pinned seq_to_head."""
    Sg = S * P  # the global sequence: rank g holds positions [g S, (g + 1) S)
    full = RNG.integers(0, 2**16, size=(B, Sg, H, D), dtype=np.uint16)
    shards = [full[:, g * S:(g + 1) * S].copy() for g in range(P)]
    sent = [oracle.split_heads(shards[g], P) for g in range(P)]  # sent[g][r]: rank g's block for rank r
    for g in range(P):
        for r in range(P):
            assert np.array_equal(sent[g][r], shards[g][:, :, r * (H // P):(r + 1) * (H // P)])
        assert np.array_equal(oracle.merge_heads(sent[g]), shards[g])
    ulysses = oracle.seq_to_head(shards, H)
    for r in range(P):
        received = np.concatenate([sent[g][r] for g in range(P)], axis=1)
        assert np.array_equal(received, ulysses[r])
    # and the way back: head_to_seq equals the block transpose followed by merge_heads on every rank
    back = oracle.head_to_seq(ulysses, Sg)
    for g in range(P):
        got = oracle.merge_heads([ulysses[r][:, g * S:(g + 1) * S] for r in range(P)])
        assert np.array_equal(got, back[g]) and np.array_equal(got, shards[g])
    # a mistake in the head offset is caught: swapping two groups breaks the identity
    if P > 1:
        swapped = list(sent[0])
        swapped[0], swapped[1] = swapped[1], swapped[0]
        assert not np.array_equal(oracle.merge_heads(swapped), shards[0])


def test_tile_list_against_nonzero():
    mask = (RNG.random((3, 7, 7)) < 0.4).astype(np.uint8)
    mask[1, 2, :] = 0
    row_ptr, col_idx = oracle.tile_list(mask)
    assert row_ptr[0] == 0 and row_ptr[-1] == int(mask.sum())
    for h in range(3):
        for i in range(7):
            r = h * 7 + i
            assert list(col_idx[row_ptr[r]:row_ptr[r + 1]]) == list(np.nonzero(mask[h, i])[0])


# ---------------------------------------------------------------------------------------------------
# Planted mistakes: a mutated copy of the oracle must fail the pins above
# ---------------------------------------------------------------------------------------------------
MUTANTS = {
    "drop_scale": ("s[j] = dot * scale;", "s[j] = dot;"),
    "transposed_key_index": ("const double* kj = J->k + (((size_t)b * S + j) * H + h) * D;",
                             "const double* kj = J->k + (((size_t)b * S + i) * H + h) * D;"),
    "causal_off_by_one": ("if (r->causal && j > i) return 0;", "if (r->causal && j >= i) return 0;"),
    "lse_drops_log": ("*lsei = m + log(l);", "*lsei = m;"),
    "merge_weight_sign": ("const double w = exp(lse_parts[p][li] - L);",
                          "const double w = exp(L - lse_parts[p][li]);"),
    "relayout_rank_index": ("const int src_rank = s / Sl, src_s = s % Sl, src_h = r * Hl + hh;",
                            "const int src_rank = s % P, src_s = s / P, src_h = r * Hl + hh;"),
    "mask_tile_transposed": ("(size_t)(i / r->tile)) * r->n_tiles + (size_t)(j / r->tile)",
                             "(size_t)(j / r->tile)) * r->n_tiles + (size_t)(i / r->tile)"),
    "bwd_drops_delta": ("const double ds = p[j] * (dp - delta);", "const double ds = p[j] * dp;"),
    "bwd_dk_unscaled": ("J->dk[IDX(k, j, d)] += ds * J->q[IDX(q, i, d)] * scale;",
                        "J->dk[IDX(k, j, d)] += ds * J->q[IDX(q, i, d)];"),
    "bwd_dv_wrong_row": ("J->dv[IDX(v, j, d)] += p[j] * J->dout[IDX(dout, i, d)];",
                         "J->dv[IDX(v, j, d)] += p[j] * J->dout[IDX(dout, j, d)];"),
}


def _pins_pass(lib):
    """A compact run of the pins above against the library at path ``lib``; False on any failure."""
    g = np.random.default_rng(7)
    B, S, H, D, T = 1, 10, 2, 4, 3
    q, k, v = (g.standard_normal((B, S, H, D)) for _ in range(3))
    nt = (S + T - 1) // T
    mask = (g.random((H, nt, nt)) < 0.5).astype(np.uint8)
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal=causal, block_mask=mask, tile=T, lib=lib)
        ob, lb = brute_force(q, k, v, lambda b, h, i, j: mask[h, i // T, j // T] != 0
                             and ((not causal) or j <= i))
        if np.max(np.abs(o - ob)) > 1e-12:
            return False
        if not np.array_equal(np.isneginf(lse), np.isneginf(lb)):
            return False
        fin = np.isfinite(lb)
        if np.max(np.abs(lse[fin] - lb[fin])) > 1e-12:
            return False
    parts = [oracle.attention(q, k, v, kv_begin=a, kv_end=e, lib=lib) for a, e in ((0, 4), (4, 10))]
    full = oracle.attention(q, k, v, lib=lib)
    mo, ml = oracle.merge([p[0] for p in parts], [p[1] for p in parts], lib=lib)
    if np.max(np.abs(mo - full[0])) > 1e-12 or np.max(np.abs(ml - full[1])) > 1e-12:
        return False
    x = g.integers(0, 255, size=(1, 8, 4, 2), dtype=np.uint8)
    outs = oracle.seq_to_head([x[:, :4].copy(), x[:, 4:].copy()], 4, lib=lib)
    if not (np.array_equal(outs[0], x[:, :, :2]) and np.array_equal(outs[1], x[:, :, 2:])):
        return False
    # backward: gradients against central differences of the forward (through the same library)
    qs, ks, vs, dos = (g.standard_normal((1, 4, 1, 3)) for _ in range(4))
    for causal in (False, True):
        grads = oracle.attention_bwd(qs, ks, vs, dos, causal=causal, lib=lib)
        for which in range(3):
            base = [qs, ks, vs]
            num = np.zeros_like(base[which])
            for idx in np.ndindex(num.shape):
                hi, lo = [t.copy() for t in base], [t.copy() for t in base]
                hi[which][idx] += 1e-6
                lo[which][idx] -= 1e-6
                lh = (dos * oracle.attention(*hi, causal=causal, lib=lib)[0]).sum()
                ll = (dos * oracle.attention(*lo, causal=causal, lib=lib)[0]).sum()
                num[idx] = (lh - ll) / 2e-6
            if np.max(np.abs(num - grads[which])) > 1e-6:
                return False
    return True


def test_pins_pass_on_the_oracle():
    assert _pins_pass(None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "sp_oracle.c")).read()
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mutant.c")
        with open(c, "w") as f:
            f.write(src.replace(old, new))
        lib = oracle.compile_source(c, os.path.join(d, "libmutant.so"))
        assert not _pins_pass(lib), f"planted mistake {name!r} went unnoticed"


# --- backward ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_attention_bwd_matches_finite_differences(causal):
    """The gradients equal central differences of L = sum(dO * O) through the forward oracle."""
    rng = np.random.default_rng(7)
    B, S, H, D = 1, 6, 2, 3
    q, k, v, do = (rng.standard_normal((B, S, H, D)) for _ in range(4))
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=causal)

    def loss(qq, kk, vv):
        return float((do * oracle.attention(qq, kk, vv, causal=causal)[0]).sum())

    eps = 1e-6
    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            args_p = [q, k, v]
            args_m = [q, k, v]
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p[which], args_m[which] = xp, xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, rtol=1e-6)


def test_attention_bwd_invariants_and_single_key():
    rng = np.random.default_rng(8)
    B, S, H, D = 2, 9, 3, 5
    q, k, v, do = (rng.standard_normal((B, S, H, D)) for _ in range(4))
    for causal in (False, True):
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=causal)
        # sum_j ds_ij = 0 for every row, so the key gradients sum to zero; rows of p sum to 1, so the value
        # gradients sum to the upstream gradients
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
        np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-12)
    # one key: o = v_0 exactly, so dv_0 = do_0 and nothing flows into q or k
    q1, k1, v1, do1 = (rng.standard_normal((1, 1, 1, 4)) for _ in range(4))
    dq, dk, dv = oracle.attention_bwd(q1, k1, v1, do1)
    np.testing.assert_allclose(dv, do1, atol=1e-15)
    assert np.all(dq == 0) and np.all(dk == 0)
    # causal: query 0 sees key 0 only, so its gradient does not reach later keys and dq_0 = 0
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal=True)
    np.testing.assert_allclose(dq[:, 0], 0.0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_bwd_rows_matches_finite_differences(causal):
    """The row-sampled gradients equal central differences of L = sum(dO * O) through the forward oracle,
    for the sampled query rows (dq) and key rows (dk, dv) of the sampled heads."""
    rng = np.random.default_rng(11)
    B, S, H, D = 2, 7, 3, 3
    q, k, v, do = (rng.standard_normal((B, S, H, D)) for _ in range(4))
    heads, q_rows, k_rows = [2, 0], [0, 4, 6], [6, 1]
    dq, dk, dv = oracle.attention_bwd_rows(q, k, v, do, heads=heads, q_rows=q_rows, k_rows=k_rows, causal=causal)

    def loss(qq, kk, vv):
        return float((do * oracle.attention(qq, kk, vv, causal=causal)[0]).sum())

    eps = 1e-6
    for x, which, rows, g in ((q, 0, q_rows, dq), (k, 1, k_rows, dk), (v, 2, k_rows, dv)):
        for b in range(B):
            for n_h, h in enumerate(heads):
                for n, r in enumerate(rows):
                    for d in range(D):
                        args_p, args_m = [q, k, v], [q, k, v]
                        xp, xm = x.copy(), x.copy()
                        xp[b, r, h, d] += eps
                        xm[b, r, h, d] -= eps
                        args_p[which], args_m[which] = xp, xm
                        num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
                        np.testing.assert_allclose(g[b, n, n_h, d], num, atol=1e-7, rtol=1e-6)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_bwd_rows_agrees_with_full_backward(causal):
    """Same numbers as the full C backward at the sampled rows (two implementations of one definition)."""
    rng = np.random.default_rng(12)
    B, S, H, D = 1, 300, 3, 16
    q, k, v, do = (rng.standard_normal((B, S, H, D)) for _ in range(4))
    heads, q_rows, k_rows = [1, 2], [0, 127, 128, 299], [0, 128, 255, 299]
    dq, dk, dv = oracle.attention_bwd_rows(q, k, v, do, heads=heads, q_rows=q_rows, k_rows=k_rows, causal=causal)
    fq, fk, fv = oracle.attention_bwd(q, k, v, do, causal=causal)
    np.testing.assert_allclose(dq, fq[:, q_rows][:, :, heads], atol=1e-11, rtol=1e-9)
    np.testing.assert_allclose(dk, fk[:, k_rows][:, :, heads], atol=1e-11, rtol=1e-9)
    np.testing.assert_allclose(dv, fv[:, k_rows][:, :, heads], atol=1e-11, rtol=1e-9)
