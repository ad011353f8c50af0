"""Shared test helpers: the error metric, the parity error log and small seeded-input builders."""
import numpy as np

# Every parity comparison that goes through check_parity() is recorded here and printed as a
# table at the end of the pytest session (tests/conftest.py), so a run's log carries the
# measured errors next to the pass/fail result.
PARITY_LOG = []


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


def error_stats(x, ref, head_axes=None, floor_frac=1e-2):
    """Error figures of one output tensor against its reference.

    rel       max|x - ref| / max|ref| (the pass metric)
    abs       max|x - ref|
    elem      max_i |x_i - ref_i| / (|ref_i| + floor), floor = floor_frac * max|ref|: the
              element-wise relative error, with small reference values measured against the floor
    head_rel  the pass metric per head (the tensor split along `head_axes`, which are kept),
              worst head: an error confined to the small-magnitude heads shows here
    """
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if x.size == 0:
        return dict(rel=0.0, abs=0.0, elem=0.0, head_rel=0.0)
    if not np.all(np.isfinite(x)):
        inf = float("inf")
        return dict(rel=inf, abs=inf, elem=inf, head_rel=inf)
    d = np.abs(x - ref)
    a = np.abs(ref)
    scale = float(a.max())
    out = dict(rel=max_rel_err(x, ref), abs=float(d.max()))
    out["elem"] = float(np.max(d / (a + floor_frac * scale))) if scale > 0 else float(d.max())
    if head_axes:
        red = tuple(i for i in range(x.ndim) if i not in head_axes)
        hd, ha = d.max(axis=red), a.max(axis=red)
        with np.errstate(divide="ignore", invalid="ignore"):
            r = np.where(ha > 0, hd / np.where(ha > 0, ha, 1.0), hd)
        out["head_rel"] = float(r.max())
    else:
        out["head_rel"] = out["rel"]
    return out


def check_parity(case: str, tensor: str, x, ref, tol: float, head_axes=None, head_tol=None):
    """Record the error figures of one output tensor and assert the pass bar max rel <= tol
    (and, when given, the per-head bar head_tol).  Returns the figures."""
    s = error_stats(x, ref, head_axes=head_axes)
    PARITY_LOG.append(dict(case=case, tensor=tensor, tol=tol, **s))
    assert s["rel"] <= tol, f"{case} {tensor}: max rel err {s['rel']:.3e} > {tol:g}"
    if head_tol is not None:
        assert s["head_rel"] <= head_tol, f"{case} {tensor}: worst head {s['head_rel']:.3e} > {head_tol:g}"
    return s


def merge_stats(items):
    """Worst case of several error_stats() results (e.g. one per step or per slice)."""
    keys = ("rel", "abs", "elem", "head_rel")
    return {k: max(s[k] for s in items) for k in keys}


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
