"""fp64 CPU oracle for the KDA recurrence -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may
import this package.  The product path (the CUDA library and its Python binding) never
does, and has no CPU fallback.

The arithmetic lives in `kda_oracle.c` (plain C, fp64, token by token; see its header
for the recurrence and the passages it follows).  This module compiles it with gcc and
wraps it with ctypes.  Inputs of any float dtype (bf16, fp32, fp64; torch or numpy) are
widened losslessly to fp64 before the call.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library next to its source; return its path."""
    with _lock:
        stale = (not os.path.exists(_LIB_PATH)
                 or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB_PATH + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def build_variant(source_text: str, out_path: str) -> ctypes.CDLL:
    """Compile a modified copy of the oracle source (used by the mutation tests)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", src, "-o", out_path,
                    "-lm"], check=True)
    return _bind(ctypes.CDLL(out_path))


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    L = ctypes.c_long
    lib.kda_oracle_forward.argtypes = [P, P, P, P, P, P, P, P, L, L, L, L, L, ctypes.c_int]
    lib.kda_oracle_forward.restype = ctypes.c_int
    if hasattr(lib, "kda_oracle_forward_states"):
        lib.kda_oracle_forward_states.argtypes = [P, P, P, P, P, P, P, P, P, L, L, L, L, L, L, ctypes.c_int]
        lib.kda_oracle_forward_states.restype = ctypes.c_int
    lib.kda_oracle_decode_step.argtypes = [P, P, P, P, P, P, P, L, L, L, L, ctypes.c_int]
    lib.kda_oracle_decode_step.restype = ctypes.c_int
    lib.kda_oracle_max_threads.argtypes = []
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    return lib


def _get_lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def max_threads() -> int:
    return int(_get_lib().kda_oracle_max_threads())


def to_f64(x) -> np.ndarray:
    """Widen a torch tensor or array to a contiguous fp64 numpy array (exact for bf16/fp32)."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q, k, v, g, beta, S0=None, nthreads: int = 0, lib: ctypes.CDLL = None):
    """Run the recurrence over [B, T, H, *] inputs; return (o [B,T,H,dv], S_T [B,H,dk,dv]) fp64."""
    lib = lib or _get_lib()
    q, k, v, g, beta, S0 = (to_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and g.shape == (B, T, H, dk)
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    o = np.zeros((B, T, H, dv), np.float64)
    ST = np.zeros((B, H, dk, dv), np.float64)
    rc = lib.kda_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                _ptr(ST), B, T, H, dk, dv, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected the shapes (rc={rc})")
    return o, ST


def prologue(q_raw, k_raw, z_g, z_beta):
    """The gate and normalisation prologue in fp64: (q, k, g, beta).

    g = -5 * sigmoid(z_g): the bounded scaled-sigmoid log-decay with lower bound -5 (skill card
    (skillsmp.com), quick facts); beta = sigmoid(z_beta) (reading: one logit per token and head);
    q, k divided by their L2 norm over the head dimension (the input recipe of the workloads; a
    zero row stays zero).
    """
    q_raw, k_raw, z_g, z_beta = (to_f64(x) for x in (q_raw, k_raw, z_g, z_beta))

    def unit(x):
        n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
        return np.divide(x, n, out=np.zeros_like(x), where=n > 0)

    g = -5.0 / (1.0 + np.exp(-z_g))
    beta = 1.0 / (1.0 + np.exp(-z_beta))
    return unit(q_raw), unit(k_raw), g, beta


def forward_fused(q_raw, k_raw, v, z_g, z_beta, S0=None, nthreads: int = 0, lib: ctypes.CDLL = None):
    """The prologue, then forward(): what the prologue-fused prefill computes."""
    q, k, g, beta = prologue(q_raw, k_raw, z_g, z_beta)
    return forward(q, k, v, g, beta, S0, nthreads=nthreads, lib=lib)


def forward_states(q, k, v, g, beta, S0=None, interval: int = 512, nthreads: int = 0,
                   lib: ctypes.CDLL = None):
    """forward() that also returns the state after every `interval` tokens.

    Returns (o [B,T,H,dv], S_T [B,H,dk,dv], S_mid [B,H,T//interval,dk,dv]) in fp64; S_mid[:, :, n]
    is the state after the first (n+1)*interval tokens.
    """
    lib = lib or _get_lib()
    q, k, v, g, beta, S0 = (to_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert interval > 0
    o = np.zeros((B, T, H, dv), np.float64)
    ST = np.zeros((B, H, dk, dv), np.float64)
    S_mid = np.zeros((B, H, T // interval, dk, dv), np.float64)
    rc = lib.kda_oracle_forward_states(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                       _ptr(o), _ptr(ST), _ptr(S_mid), int(interval), B, T, H, dk, dv,
                                       int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected the shapes (rc={rc})")
    return o, ST, S_mid


def decode_step(q, k, v, g, beta, S: np.ndarray, nthreads: int = 0, lib: ctypes.CDLL = None):
    """One token for every (batch, head): updates S [B,H,dk,dv] (fp64, in place); returns o [B,H,dv]."""
    lib = lib or _get_lib()
    q, k, v, g, beta = (to_f64(x) for x in (q, k, v, g, beta))
    assert S.dtype == np.float64 and S.flags["C_CONTIGUOUS"]
    B, H, dk = q.shape
    dv = v.shape[-1]
    assert S.shape == (B, H, dk, dv)
    o = np.zeros((B, H, dv), np.float64)
    rc = lib.kda_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                    B, H, dk, dv, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected the shapes (rc={rc})")
    return o
