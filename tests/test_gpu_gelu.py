"""The device GeLU and its derivative (what the FC1 epilogue applies and the
FC2-dgrad epilogue differentiates) against the exact definitions in fp64:
GeLU(x) = x Phi(x), GeLU'(x) = Phi(x) + x phi(x) (rkmt.cn guide, section 3.1).
The device evaluates Phi through a rational approximation of erf whose error
is at most 1.5e-7; fp32 rounding adds a few ulp, hence the bound below."""
import math

import numpy as np
import pytest
import torch

from tensor_transformer_layer_tp_b200 import binding as B

pytestmark = pytest.mark.gpu


def _exact(x):
    x = np.asarray(x, dtype=np.float64)
    cdf = 0.5 * (1.0 + np.vectorize(math.erf)(x / math.sqrt(2.0)))
    pdf = np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    return x * cdf, cdf + x * pdf


def test_gelu_and_derivative_match_the_definition():
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.linspace(-12.0, 12.0, 48001),
                   3.0 * torch.randn(50000, generator=g),
                   torch.tensor([0.0, -0.0, 1e-30, -1e-30, 1e-3, -1e-3, 40.0, -40.0])])
    xd = x.cuda()
    y, dy = torch.empty_like(xd), torch.empty_like(xd)
    B.tp_gelu_eval(xd, y, dy)
    torch.cuda.synchronize()
    ref_y, ref_dy = _exact(x.numpy())
    xa = np.abs(x.numpy().astype(np.float64))
    err_y = np.abs(y.cpu().numpy() - ref_y)
    err_dy = np.abs(dy.cpu().numpy() - ref_dy)
    assert np.all(np.isfinite(y.cpu().numpy())) and np.all(np.isfinite(dy.cpu().numpy()))
    assert np.max(err_y / (1e-7 + 5e-7 * xa)) <= 1.0, f"GeLU max err {err_y.max():.3e}"
    assert np.max(err_dy / (1e-6 + 5e-7 * xa)) <= 1.0, f"GeLU' max err {err_dy.max():.3e}"
