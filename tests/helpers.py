"""Shared test utilities: dtype conversion and the parity tolerances.

Tolerances (from the stated accuracy target of the layer and loss):
  * every bf16-in / fp32-accumulate output tensor: max|gpu - ref| <= 2e-2 * max|ref|
  * the fp32 loss of the cross-entropy: relative error <= 1e-5
"""
import numpy as np
import torch

TENSOR_TOL = 2e-2
LOSS_RTOL = 1e-5


def f64(t):
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").double().numpy()


def max_rel_err(got, ref):
    got, ref = f64(got), f64(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / max(scale, 1e-30))


def assert_close(name, got, ref, tol=TENSOR_TOL):
    got64 = f64(got)
    assert np.all(np.isfinite(got64)), f"{name}: non-finite values"
    err = max_rel_err(got64, ref)
    assert err <= tol, f"{name}: max|err|/max|ref| = {err:.3e} > {tol:.1e}"
    return err


def to_dev(t, device="cuda"):
    return t.to(device).contiguous()
