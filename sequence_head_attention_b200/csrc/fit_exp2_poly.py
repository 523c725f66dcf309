"""Minimax (Remez exchange) fit of 2^f on [-1/2, 1/2] with relative-error weight, for the part of the
softmax exponentials the attention kernel evaluates on the FMA pipe instead of the MUFU unit.

Method: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (an exact split in fp32 for the
arguments the kernel sees after clamping, x in [-125, 8]); 2^f is replaced by the polynomial c0 + c1 f + ... + cd f^d
whose maximum relative error on [-1/2, 1/2] is minimal (Remez's second algorithm: solve for the
coefficients and the levelled error on d + 2 reference points, move the reference to the extrema of the
error curve, repeat).

Run it to print the fp32 coefficients written into attn_fwd.cu and the error bound the tests check:
    python sequence_head_attention_b200/csrc/fit_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(degree: int, iters: int = 60, grid: int = 200001):
    """Coefficients c0..c_degree minimising max |p(f)/2^f - 1| on [-1/2, 1/2], as float64."""
    a, b = -0.5, 0.5
    xs = np.linspace(a, b, grid)
    n = degree + 1  # unknown coefficients; the reference has n + 1 points
    k = np.arange(n + 1)
    ref = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - k) / n)
    coef = None
    for _ in range(iters):
        # sum_j c_j x_i^j - (-1)^i E 2^x_i = 2^x_i   (relative error levelled at +-E)
        A = np.zeros((n + 1, n + 1))
        rhs = np.exp2(ref)
        for i, x in enumerate(ref):
            A[i, :n] = [x ** j for j in range(n)]
            A[i, n] = -((-1) ** i) * np.exp2(x)
        coef = np.linalg.solve(A, rhs)[:n]
        err = np.polyval(coef[::-1], xs) / np.exp2(xs) - 1.0
        # new reference: one point of largest |err| per run of equal sign, n + 1 runs
        idx = [0] + [i for i in range(1, grid - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0]
        idx.append(grid - 1)
        runs = []
        for i in idx:
            if runs and np.sign(err[runs[-1]]) == np.sign(err[i]):
                if abs(err[i]) > abs(err[runs[-1]]):
                    runs[-1] = i
            else:
                runs.append(i)
        while len(runs) > n + 1:
            runs.pop(0 if abs(err[runs[0]]) < abs(err[runs[-1]]) else -1)
        if len(runs) < n + 1:
            break
        ref = xs[runs]
    return coef


def eval_fp32(coef32, x):
    """The kernel's evaluation in fp32: n = round(x), f = x - n, Horner with fused multiply-adds (each
    fma rounded once to fp32), scale by 2^n through the exponent field."""
    x = np.asarray(x, dtype=np.float32)
    x = np.maximum(x, np.float32(-125.0))
    n = np.rint(x).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(coef32[-1])
    for c in coef32[-2::-1]:
        p = (np.float64(p) * np.float64(f) + np.float64(c)).astype(np.float32)
    bits = p.view(np.int32) + (n.astype(np.int32) << 23)
    return bits.view(np.float32)


def max_rel_error(coef32, lo=-30.0, hi=8.0, n=2_000_001):
    x = np.linspace(lo, hi, n).astype(np.float32)
    y = eval_fp32(coef32, x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(y / ref - 1.0)))


if __name__ == "__main__":
    d = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez_exp2(d)
    c32 = c.astype(np.float32)
    print("degree", d)
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v):.9e}f  ({v.view(np.uint32):#010x})")
    print("max relative error (fp32 evaluation, x in [-30, 8]):", max_rel_error(c32))
