"""Shared helpers of the tests: error metrics and layout mapping (no arithmetic of
the method lives here)."""
import numpy as np
import torch

# max relative error, tensor-normalised: max|gpu - ref| / max|ref|
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


def np64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def rel_err(gpu, ref):
    g, r = np64(gpu), np64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    den = np.max(np.abs(r))
    if den == 0.0:
        return float(np.max(np.abs(g)))
    return float(np.max(np.abs(g - r)) / den)


def assert_close(name, gpu, ref, dtype):
    err = rel_err(gpu, ref)
    assert err <= TOL[dtype], f"{name}: max rel err {err:.3e} > {TOL[dtype]:.1e}"
    return err
