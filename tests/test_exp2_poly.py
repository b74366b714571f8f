"""The FMA-pipe 2^x approximation used by the prefill softmax.

CPU: the coefficients in csrc/common.cuh are the ones the committed fitting
script produces, and the fit meets its error bound.  GPU: the device
evaluation against torch.exp2 (CUDA's exp2f) over the range the softmax uses.
"""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coeffs_in_source():
    with open(os.path.join(ROOT, "attention_varlen_gqa_b200", "csrc", "common.cuh")) as f:
        text = f.read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1)) for i in range(4)]


def test_coefficients_match_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fit", os.path.join(ROOT, "attention_varlen_gqa_b200", "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, err = fit.fit()
    assert err < 8e-5
    src = _coeffs_in_source()
    assert np.allclose(np.float32(c), np.float32(src), rtol=0, atol=0)


def test_cubic_error_bound_fp32():
    c = np.float32(_coeffs_in_source())
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5


@pytest.mark.gpu
def test_device_polynomial_against_exp2f():
    import torch
    import attention_varlen_gqa_b200 as A
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20, device="cuda"),
                   torch.randn(1 << 16, device="cuda") * 4.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.5, -0.25], device="cuda")])
    y = A.attn_selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel
    # below the clamp the result is 2^-125-sized, never NaN, negative or denormal
    z = A.attn_selftest_exp2(torch.tensor([-200.0, -float("inf"), -127.0], device="cuda"))
    assert torch.all(torch.isfinite(z)) and torch.all(z >= 1.1754944e-38) and torch.all(z < 4e-38)
