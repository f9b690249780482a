"""Shared helpers of the tests (no method arithmetic)."""
import numpy as np


def normwise_err(got, ref):
    """max_i |g_i - r_i| / max_i |r_i|."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-30))


def dev(a, device):
    from int4_weight_only_02_b200.runtime import to_device
    return to_device(np.asarray(a), device)
