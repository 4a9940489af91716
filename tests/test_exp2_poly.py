"""The attention kernel's FMA-pipe exponential: its polynomial is the fit the
committed script produces, and the Cody-Waite reconstruction keeps the
relative error under 7.5e-5 over the softmax's input range. The GPU test
checks the device code itself against fp64 and against CUDA's exp2."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_video_lcsa_b200", "csrc")
BOUND = 7.5e-5


def kernel_coefficients():
    text = open(os.path.join(CSRC, "k3_attention_tc.cu")).read()
    return np.array([float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f" % k, text).group(1)) for k in range(4)],
                    dtype=np.float32)


def fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def emulate(x, c):
    """fp32 emulation of exp2_poly (shifter rounding, f, Horner, exponent add)."""
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shifter = np.float32(12582912.0)
    t = (x + shifter).astype(np.float32)
    n = (t - shifter).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full(x.shape, c[3], dtype=np.float32)
    for k in (2, 1, 0):
        p = (p.astype(np.float64) * f + c[k]).astype(np.float32)     # fma: one rounding
    ni = (t.view(np.uint32) - np.uint32(0x4B400000)).astype(np.uint32)
    return (p.view(np.uint32) + (ni << np.uint32(23))).view(np.float32)


def test_kernel_holds_the_fitted_polynomial():
    np.testing.assert_array_equal(kernel_coefficients(), fit_module().fit())


def test_reconstruction_error_bound():
    c = kernel_coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), np.linspace(-1.0, 1.0, 100001)]).astype(np.float32)
    y = emulate(x, c)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert np.abs(y / ref - 1).max() < BOUND


@pytest.mark.gpu
def test_device_exponential_matches_fp64_and_cuda():
    import torch
    import block_sparse_video_lcsa_b200 as L
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.linspace(-1.0, 1.0, 1 << 16),
                   torch.tensor([0.0, -0.5, 0.5, 7.999, -124.9])]).float().cuda()
    y = torch.empty_like(x)
    L.lcsa_selftest_exp2(x, y)
    torch.cuda.synchronize()
    yd = y.double().cpu().numpy()
    ref = np.exp2(x.double().cpu().numpy())
    assert np.abs(yd / ref - 1).max() < BOUND
    cuda = torch.exp2(x).double().cpu().numpy()
    assert np.abs(yd / cuda - 1).max() < BOUND + 1e-6
    np.testing.assert_allclose(y.cpu().numpy(), emulate(x.cpu().numpy(), kernel_coefficients()), rtol=3e-7, atol=0)
