"""Shared helpers of the parity tests (comparison against the oracle, tolerances)."""
import numpy as np
import torch

# max|gpu - ref| <= TOL * max|ref| per tensor
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref))
    if scale == 0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref)) / scale)


def assert_close(name, got, ref, dtype):
    err = rel_err(got, ref)
    assert np.all(np.isfinite(np.asarray(got, np.float64))), f"{name}: non-finite output"
    assert err <= TOL[dtype], f"{name}: max|gpu-ref|/max|ref| = {err:.3e} > {TOL[dtype]:.0e}"
    return err
