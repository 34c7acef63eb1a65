"""Shared test utilities (no method arithmetic)."""

import numpy as np

TOL_BF16 = 2e-2   # relative Frobenius error, bf16 compute paths
TOL_FP32 = 1e-4   # relative Frobenius error, fp32 compute paths


def rel_fro(got, ref, axis=(-2, -1)):
    """max over the batch of ||got - ref||_F / ||ref||_F."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.sqrt(np.sum((got - ref) ** 2, axis=axis))
    den = np.sqrt(np.sum(ref ** 2, axis=axis))
    return float(np.max(num / np.maximum(den, 1e-300)))


def to_np(t):
    return t.detach().to("cpu").double().numpy()
