"""The FMA-pipe exponential of the attention kernel: its coefficients are the minimax fit the committed
fitter produces, its fp32 evaluation meets the fit's error bound, and on the GPU it agrees with CUDA's
exp2f within that bound."""
import importlib.util
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sequence_head_attention_b200", "csrc")
BOUND = 8e-5  # max relative error of the fp32 evaluation (the fit gives 7.5e-5)


def _fitter():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "sp_ptx.cuh")).read()
    body = src[src.index("exp2_poly2"):]
    return [float(re.search(rf"const f2 c{i} = {{([-0-9.e+]+)f,", body).group(1)) for i in range(4)]


def test_kernel_coefficients_are_the_minimax_fit():
    fit = _fitter()
    c = fit.remez_exp2(3).astype(np.float32)
    k = np.array(_kernel_coefficients(), dtype=np.float32)
    assert np.allclose(c, k, rtol=2e-7, atol=0), (c, k)


def test_fp32_evaluation_error_bound():
    fit = _fitter()
    k = np.array(_kernel_coefficients(), dtype=np.float32)
    assert fit.max_rel_error(k) < BOUND
    # and the fit is a real minimax: a plain Taylor cubic is several times worse on the same interval
    taylor = np.array([1.0, np.log(2), np.log(2) ** 2 / 2, np.log(2) ** 3 / 6], dtype=np.float32)
    assert fit.max_rel_error(taylor) > 5 * fit.max_rel_error(k)


@pytest.mark.gpu
def test_gpu_polynomial_against_cuda_exp2f():
    from sequence_head_attention_b200 import spattn
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 7.99, -124.6, 1e-7])])
    if x.numel() % 2:
        x = torch.cat([x, torch.tensor([0.0])])
    xd = x.cuda()
    y = torch.empty_like(xd)
    spattn.sp_debug_exp2_poly(xd, y)
    ref = torch.exp2(xd.double())
    rel = ((y.double() - ref) / ref).abs()
    assert float(rel.max()) < BOUND
    # inputs below the clamp give 2^-125 (tiny, finite), -inf included
    z = torch.tensor([-float("inf"), -1000.0], device="cuda")
    yz = torch.empty_like(z)
    spattn.sp_debug_exp2_poly(z, yz)
    assert torch.all(torch.isfinite(yz)) and torch.all(yz < 1e-37) and torch.all(yz >= 0)
