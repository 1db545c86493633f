"""Comparison helpers of the parity tests.

Tolerance (per output tensor, GPU result g against the fp64 oracle r):
    max|g - r| / max|r|  <=  max_rel      (1e-2 for bf16, 3e-2 fp8 cache)
    mean|g - r|          <=  mae          (2e-3)
"""
import numpy as np

BF16_MAX_REL, BF16_MAE = 1e-2, 2e-3
FP8_MAX_REL = 3e-2


def errors(g, r):
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(fin, np.isfinite(g)), "non-finite pattern differs"
    err = np.abs(g[fin] - r[fin])
    scale = np.max(np.abs(r[fin])) if fin.any() else 1.0
    return (float(err.max() / scale) if err.size else 0.0, float(err.mean()) if err.size else 0.0)


def assert_close(name, g, r, max_rel=BF16_MAX_REL, mae=BF16_MAE):
    mr, ma = errors(g, r)
    assert mr <= max_rel and ma <= mae, (
        f"{name}: max rel err {mr:.3e} (limit {max_rel}), mean abs err {ma:.3e} (limit {mae})")
    return mr, ma


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (the quantum of x's binade)."""
    x = np.abs(np.asarray(x, np.float64))
    _, k = np.frexp(np.where(x > 0, x, 1.0))
    return np.ldexp(1.0, (k - 8).astype(np.int64))
