"""Shared test helpers: tolerance checks against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation; the P probabilities are rounded to bf16 before P V):
  O:   max |x - y| <= 2e-2 and ||x - y||_2 / ||y||_2 <= 5e-3
  LSE: max |x - y| <= 1e-3 over finite entries, and -inf exactly where the oracle has -inf.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def to64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def metrics(o, o_ref, lse=None, lse_ref=None):
    o, o_ref = to64(o), to64(o_ref)
    d = o - o_ref
    m = {"max_abs": float(np.max(np.abs(d))) if d.size else 0.0,
         "rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(o_ref), 1e-30)) if d.size else 0.0}
    if lse is not None:
        lse, lse_ref = to64(lse), to64(lse_ref)
        fin = np.isfinite(lse_ref)
        m["lse_inf_match"] = bool(np.array_equal(np.isneginf(lse), np.isneginf(lse_ref)))
        m["lse_finite"] = bool(np.all(np.isfinite(lse[fin])))
        m["lse_max_abs"] = float(np.max(np.abs(lse[fin] - lse_ref[fin]))) if fin.any() else 0.0
    return m


def assert_close(o, o_ref, lse=None, lse_ref=None, o_max_abs=O_MAX_ABS, o_rel_l2=O_REL_L2,
                 lse_max_abs=LSE_MAX_ABS):
    m = metrics(o, o_ref, lse, lse_ref)
    assert np.all(np.isfinite(to64(o))), m
    assert m["max_abs"] <= o_max_abs, m
    assert m["rel_l2"] <= o_rel_l2, m
    if lse is not None:
        assert m["lse_inf_match"], m
        assert m["lse_finite"], m
        assert m["lse_max_abs"] <= lse_max_abs, m
    return m
