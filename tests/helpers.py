"""Shared test helpers: the error metric and small seeded-input builders."""
import numpy as np


def max_rel_err(x, ref) -> float:
    """max_i |x_i - ref_i| / max_i |ref_i| over a whole output tensor.

    When the reference is identically zero the result must be exactly zero too; the
    function then returns max|x| (so any nonzero output fails a tolerance check of 0).
    """
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if x.size == 0:
        return 0.0
    if not np.all(np.isfinite(x)):
        return float("inf")
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(x - ref))
    if scale == 0.0:
        return float(err)
    return float(err / scale)


def unit_rows(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_problem(rng, B, T, H, dk, dv, s0=True, g_lo=-5.0):
    """fp64 inputs with the recipe's distributions (unit q/k, beta in (0,1), g in [g_lo, 0))."""
    q = unit_rows(rng, (B, T, H, dk))
    k = unit_rows(rng, (B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    g = g_lo / (1.0 + np.exp(-rng.standard_normal((B, T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None
    return q, k, v, g, beta, S0
