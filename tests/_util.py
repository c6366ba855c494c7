"""Shared helpers of the tests: error metrics and layout mapping (no arithmetic of
the method lives here)."""
import json
import os

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


def log_parity(name, err, tol):
    """Append one measured error to the JSON-lines file named by SMOE_PARITY_LOG (if set)."""
    path = os.environ.get("SMOE_PARITY_LOG")
    if not path:
        return
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(path, "a") as fh:
        fh.write(json.dumps({"test": test, "name": name, "err": err, "tol": tol}) + "\n")


def assert_close(name, gpu, ref, dtype):
    err = rel_err(gpu, ref)
    log_parity(name, err, TOL[dtype])
    assert err <= TOL[dtype], f"{name}: max rel err {err:.3e} > {TOL[dtype]:.1e}"
    return err
