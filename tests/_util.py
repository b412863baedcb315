"""Helpers shared by the GPU parity tests (comparison only; no arithmetic of the method)."""
import numpy as np
import torch

TOL_BF16 = 2e-2   # max|gpu - oracle| / max|oracle| for bf16 inputs
TOL_F32 = 1e-4    # ... for fp32 inputs


def f64(t):
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    den = np.max(np.abs(ref))
    if den == 0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(gpu - ref)) / den)


def tol_for(dtype):
    return TOL_BF16 if dtype == torch.bfloat16 else TOL_F32


def cuda(x):
    return None if x is None else x.to("cuda").contiguous()
