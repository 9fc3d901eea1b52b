"""Comparison helpers for GPU-vs-oracle parity.

The bar for floating-point outputs is the one stated for this layer: element-wise
max-abs error <= 2e-2 and relative L2 error <= 5e-3 against the fp64 oracle on the same
seeded bf16 inputs.
"""
import numpy as np

MAX_ABS = 2e-2
REL_L2 = 5e-3


def errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    diff = g - r
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(r.ravel()))
    rel = float(np.linalg.norm(diff.ravel()) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_parity(gpu, ref, what="", max_abs=MAX_ABS, rel_l2=REL_L2):
    g = np.asarray(gpu, dtype=np.float64)
    assert np.all(np.isfinite(g)), "%s: non-finite values in the GPU result" % what
    ma, rl = errors(g, ref)
    assert ma <= max_abs and rl <= rel_l2, \
        "%s: max-abs %.3e (bar %.1e), rel-L2 %.3e (bar %.1e)" % (what, ma, max_abs, rl, rel_l2)
    return ma, rl


def to_np(t):
    import torch
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else \
        t.detach().cpu().numpy()
