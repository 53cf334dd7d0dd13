"""Helpers for GPU-vs-oracle comparisons (no arithmetic of the method here).

Error measure: normwise relative error max|x - ref| / max|ref| over a tensor.
Tolerances: fp32-input path 1e-4 (o and state); bf16-input path 1e-2 for o
and 5e-3 for the final state.
"""
import numpy as np
import torch

TOL_F32 = 1e-4
TOL_BF16_O = 1e-2
TOL_BF16_STATE = 5e-3


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def normwise(x, ref):
    x, ref = to64(x), to64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.isfinite(x).all(), "non-finite values in GPU result"
    den = np.abs(ref).max()
    num = np.abs(x - ref).max()
    return float(num / den) if den > 0 else float(num)


def assert_close(x, ref, tol, what):
    e = normwise(x, ref)
    assert e <= tol, "%s: normwise relative error %.3e > %.1e" % (what, e, tol)
    return e
