"""Comparison helpers shared by the parity tests."""
import numpy as np
import torch


def max_rel(gpu, ref):
    """max_i |g_i - o_i| / max_i |o_i| over one output tensor; +inf if the GPU
    result holds a non-finite value."""
    g = gpu.detach().to("cpu", torch.float64).numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    o = np.asarray(ref, dtype=np.float64)
    assert g.shape == o.shape, (g.shape, o.shape)
    if g.size == 0:
        return 0.0
    if not np.all(np.isfinite(g)):
        return float("inf")
    scale = np.max(np.abs(o))
    if scale == 0:
        return float(np.max(np.abs(g)))
    return float(np.max(np.abs(g - o)) / scale)


def assert_close(name, gpu, ref, tol):
    e = max_rel(gpu, ref)
    assert e <= tol, f"{name}: max relative error {e:.3e} > {tol:.1e}"
    return e
