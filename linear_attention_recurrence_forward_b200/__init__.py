"""Python binding of the B200 KDA recurrence library (ctypes over the C ABI in include/kda.h).

Argument marshalling only: every step of the computation runs in the CUDA kernels of
libkda_b200.so.  There is no CPU fallback; if the library is missing or a call fails,
these functions raise.

    from linear_attention_recurrence_forward_b200 import kda_forward_chunked, kda_decode_step
    o, S_T = kda_forward_chunked(q, k, v, g, beta, S0)        # prefill, torch CUDA tensors
    o, S_T, S_mid = kda_forward_chunked_states(q, k, v, g, beta, S0, interval=512)
    o, S_T = kda_forward_chunked_host(q_cpu, k_cpu, v_cpu, g_cpu, beta_cpu, S0_cpu)  # host tensors in and out
    o = kda_decode_step(q, k, v, g, beta, S)                   # one token, S updated in place

Layouts (contiguous): q, k, g [B, T, H, dk]; v, o [B, T, H, dv]; beta [B, T, H];
states [B, H, dk, dv] fp32.  Decode drops the T axis.  dtype: bf16 or fp32 (all of q, k,
v, g, beta share it; o gets it too).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "kda_forward_chunked",
    "kda_forward_chunked_states",
    "kda_forward_chunked_host",
    "kda_forward_chunked_host_noalloc",
    "host_workspace_bytes",
    "kda_decode_step",
    "kda_forward_varlen",
    "kda_forward_chunked_fused",
    "kda_decode_step_paged",
    "kda_state_compose",
    "kda_output_correct",
    "kda_get_device_status",
    "kda_status_string",
    "kda_debug_set_wait_fault",
    "KdaError",
    "lib",
    "LIB_PATH",
    "STATUS",
    "IMPL",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda_b200.so")

STATUS = {
    "KDA_OK": 0,
    "KDA_ERR_INVALID_ARG": -1,
    "KDA_ERR_UNSUPPORTED": -2,
    "KDA_ERR_MISALIGNED": -3,
    "KDA_ERR_CUDA": -4,
    "KDA_ERR_TIMEOUT": -5,
}
DTYPE = {torch.bfloat16: 0, torch.float32: 1}
IMPL = {"auto": 0, "tcgen05": 1, "simt": 2}

_lib: Optional[ctypes.CDLL] = None


class KdaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {kda_status_string(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it first (python -m linear_attention_recurrence_forward_b200.build "
                "or __graft_entry__.build()); there is no fallback implementation")
        L = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        L.kda_forward_chunked.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P]
        L.kda_forward_chunked.restype = I
        L.kda_forward_chunked_impl.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        L.kda_forward_chunked_impl.restype = I
        L.kda_forward_chunked_states.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P]
        L.kda_forward_chunked_states.restype = I
        L.kda_forward_chunked_host.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, ctypes.c_size_t, I, P]
        L.kda_forward_chunked_host.restype = I
        L.kda_forward_chunked_host_noalloc.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        L.kda_forward_chunked_host_noalloc.restype = I
        L.kda_forward_chunked_host_workspace.argtypes = [I, I, I, I, I]
        L.kda_forward_chunked_host_workspace.restype = ctypes.c_size_t
        L.kda_state_compose.argtypes = [P, P, P, P, I, I, I, P]
        L.kda_state_compose.restype = I
        L.kda_output_correct.argtypes = [P, P, P, P, I, I, I, I, I, I, P]
        L.kda_output_correct.restype = I
        L.kda_forward_chunked_fused.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        L.kda_forward_chunked_fused.restype = I
        L.kda_forward_varlen.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, P]
        L.kda_forward_varlen.restype = I
        L.kda_decode_step_paged.argtypes = [P, P, P, P, P, P, I, P, P, I, I, I, I, I, P]
        L.kda_decode_step_paged.restype = I
        L.kda_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
        L.kda_decode_step.restype = I
        L.kda_get_device_status.argtypes = [P]
        L.kda_get_device_status.restype = I
        L.kda_status_string.argtypes = [I]
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_version.argtypes = []
        L.kda_version.restype = I
        L.kda_debug_set_wait_fault.argtypes = [I, ctypes.c_ulonglong]
        L.kda_debug_set_wait_fault.restype = I
        _lib = L
    return _lib


def kda_status_string(status: int) -> str:
    return lib().kda_status_string(int(status)).decode()


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _check(t: torch.Tensor, name: str, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def kda_forward_chunked(q, k, v, g, beta, S0=None, *, o=None, S_T=None, return_state: bool = True,
                        impl: str = "auto", stream=None):
    """Prefill over [B, T, H, *] CUDA tensors.  Returns (o, S_T) (S_T None if not requested).

    S_T may be passed in (and may be S0 itself for an in-place state carry).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t, shape in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                           ("g", g, (B, T, H, dk)), ("beta", beta, (B, T, H))):
        _check(t, name, shape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _check(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_forward_chunked_impl(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                            _ptr(o), _ptr(S_T), B, T, H, dk, dv, DTYPE[dt], IMPL[impl],
                                            _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_forward_chunked", rc)
    return o, S_T


def host_workspace_bytes(T: int, H: int, dk: int = 128, dv: int = 128, dtype=torch.bfloat16) -> int:
    """Bytes of device workspace kda_forward_chunked_host needs for T tokens and H heads."""
    if dtype not in DTYPE:
        raise ValueError(f"unsupported dtype {dtype}")
    n = lib().kda_forward_chunked_host_workspace(int(T), int(H), int(dk), int(dv), DTYPE[dtype])
    if n == 0:
        raise ValueError(f"unsupported sizes T={T} H={H} dk={dk} dv={dv}")
    return int(n)


def kda_forward_chunked_host(q, k, v, g, beta, S0=None, *, o=None, S_T=None, return_state: bool = True,
                             workspace=None, impl: str = "auto", stream=None, device=None):
    """Prefill over [B, T, H, *] HOST (CPU) tensors, outputs in host memory.

    The library copies the inputs to the GPU segment by segment, runs the prefill and copies o
    and S_T back, overlapping the copies with the kernels; o and S_T equal kda_forward_chunked's
    bitwise.  Pinned inputs make the copies asynchronous; outputs allocated here are pinned.
    The call is asynchronous on `stream`: read o and S_T after synchronizing it.  `workspace` is
    a CUDA uint8 tensor of at least host_workspace_bytes(T, H, dk, dv, dtype) bytes (allocated on
    `device` if not given).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    cpu = torch.device("cpu")
    for name, t, shape in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                           ("g", g, (B, T, H, dk)), ("beta", beta, (B, T, H))):
        _check(t, name, shape, dt, cpu)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, cpu)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, pin_memory=True)
    else:
        _check(o, "o", (B, T, H, dv), dt, cpu)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=True)
    elif S_T is not None:
        _check(S_T, "S_T", (B, H, dk, dv), torch.float32, cpu)
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    nbytes = host_workspace_bytes(T, H, dk, dv, dt)
    own_workspace = workspace is None
    if own_workspace:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    elif not (isinstance(workspace, torch.Tensor) and workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    with torch.cuda.device(workspace.device):
        rc = lib().kda_forward_chunked_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(o),
                                            _ptr(S_T), B, T, H, dk, dv, DTYPE[dt], _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), IMPL[impl],
                                            _stream_handle(stream))
        if rc != 0:
            raise KdaError("kda_forward_chunked_host", rc)
        if own_workspace and stream is not None:
            workspace.record_stream(stream)   # not reused before the call's work on `stream` is done
    return o, S_T


def kda_forward_chunked_host_noalloc(q, k, v, g, beta, S0=None, *, o=None, S_T=None, return_state: bool = True,
                                     impl: str = "auto", stream=None, device=None):
    """kda_forward_chunked_host without a workspace: the library stages the work through its own fixed
    device scratch (KDA_NOALLOC_SCRATCH_BYTES per device), so nothing is allocated on the device.
    Host tensors in, host tensors out (outputs allocated here are pinned); o and S_T equal
    kda_forward_chunked_host's bitwise.  Calls whose work overlaps on the GPU share the scratch and
    race: keep them in order on one stream.  Read o and S_T after synchronizing `stream`.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    cpu = torch.device("cpu")
    for name, t, shape in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                           ("g", g, (B, T, H, dk)), ("beta", beta, (B, T, H))):
        _check(t, name, shape, dt, cpu)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, cpu)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, pin_memory=True)
    else:
        _check(o, "o", (B, T, H, dv), dt, cpu)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=True)
    elif S_T is not None:
        _check(S_T, "S_T", (B, H, dk, dv), torch.float32, cpu)
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(device):
        rc = lib().kda_forward_chunked_host_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                                    _ptr(o), _ptr(S_T), B, T, H, dk, dv, DTYPE[dt], IMPL[impl],
                                                    _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_forward_chunked_host_noalloc", rc)
    return o, S_T


def kda_forward_chunked_states(q, k, v, g, beta, S0=None, *, interval: int = 512, o=None, S_T=None,
                               S_mid=None, impl: str = "auto", stream=None):
    """Prefill that also returns the state after every `interval` tokens (a multiple of 64).

    Returns (o, S_T, S_mid) with S_mid [B, H, T // interval, dk, dv] fp32: S_mid[:, :, n] is the
    state after the first (n + 1) * interval tokens.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t, shape in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                           ("g", g, (B, T, H, dk)), ("beta", beta, (B, T, H))):
        _check(t, name, shape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    n_mid = T // interval if interval > 0 else 0
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    else:
        _check(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    if S_mid is None:
        S_mid = torch.empty((B, H, n_mid, dk, dv), dtype=torch.float32, device=dev)
    else:
        _check(S_mid, "S_mid", (B, H, n_mid, dk, dv), torch.float32, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_forward_chunked_states(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                              _ptr(o), _ptr(S_T), _ptr(S_mid) if n_mid > 0 else None,
                                              int(interval), B, T, H, dk, dv, DTYPE[dt], IMPL[impl],
                                              _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_forward_chunked_states", rc)
    return o, S_T, S_mid


def kda_decode_step(q, k, v, g, beta, S, *, o=None, stream=None):
    """One token for every (b, h).  q, k, g [B, H, dk]; v [B, H, dv]; beta [B, H]; S updated in place."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t, shape in (("q", q, (B, H, dk)), ("k", k, (B, H, dk)), ("v", v, (B, H, dv)),
                           ("g", g, (B, H, dk)), ("beta", beta, (B, H))):
        _check(t, name, shape, dt, dev)
    _check(S, "S", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, H, dv), dt, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(o),
                                   B, H, dk, dv, DTYPE[dt], _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_decode_step", rc)
    return o


def kda_forward_chunked_fused(q_raw, k_raw, v, z_g, z_beta, S0=None, *, o=None, S_T=None,
                              return_state: bool = True, impl: str = "auto", stream=None):
    """Prefill with the prologue in the kernels: g = -5 sigmoid(z_g), beta = sigmoid(z_beta), q and k
    L2-normalised over the head dimension.  Same layouts as kda_forward_chunked."""
    B, T, H, dk = q_raw.shape
    dv = v.shape[-1]
    dev, dt = q_raw.device, q_raw.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t, shape in (("q_raw", q_raw, (B, T, H, dk)), ("k_raw", k_raw, (B, T, H, dk)),
                           ("v", v, (B, T, H, dv)), ("z_g", z_g, (B, T, H, dk)), ("z_beta", z_beta, (B, T, H))):
        _check(t, name, shape, dt, dev)
    if S0 is not None:
        _check(S0, "S0", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, T, H, dv), dt, dev)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _check(S_T, "S_T", (B, H, dk, dv), torch.float32, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_forward_chunked_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(z_g), _ptr(z_beta), _ptr(S0),
                                             _ptr(o), _ptr(S_T), B, T, H, dk, dv, DTYPE[dt], IMPL[impl],
                                             _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_forward_chunked_fused", rc)
    return o, S_T


def kda_forward_varlen(q, k, v, g, beta, cu_seqlens, S0=None, *, o=None, S_T=None, return_state: bool = True,
                       impl: str = "auto", stream=None):
    """Prefill over packed sequences: q, k, g [T_total, H, dk]; v [T_total, H, dv]; beta [T_total, H];
    cu_seqlens int32 [N + 1] on the device (sequence n = tokens cu_seqlens[n] .. cu_seqlens[n+1]-1).
    States [N, H, dk, dv] fp32.  Returns (o [T_total, H, dv], S_T or None).
    """
    T_total, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.shape[0] - 1
    dev, dt = q.device, q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t, shape in (("q", q, (T_total, H, dk)), ("k", k, (T_total, H, dk)), ("v", v, (T_total, H, dv)),
                           ("g", g, (T_total, H, dk)), ("beta", beta, (T_total, H))):
        _check(t, name, shape, dt, dev)
    _check(cu_seqlens, "cu_seqlens", (N + 1,), torch.int32, dev)
    if S0 is not None:
        _check(S0, "S0", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty((T_total, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (T_total, H, dv), dt, dev)
    if S_T is None and return_state:
        S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _check(S_T, "S_T", (N, H, dk, dv), torch.float32, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), _ptr(S0),
                                      _ptr(o), _ptr(S_T), N, T_total, H, dk, dv, DTYPE[dt], IMPL[impl],
                                      _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_forward_varlen", rc)
    return o, S_T


def kda_decode_step_paged(q, k, v, g, beta, S_pool, slots, *, o=None, stream=None):
    """One token per sequence with the states in a pool: S_pool [n_slots, H, dk, dv] fp32 (updated in
    place), slots int32 [B] on the device (sequence b uses S_pool[slots[b]]; negative = skip)."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t, shape in (("q", q, (B, H, dk)), ("k", k, (B, H, dk)), ("v", v, (B, H, dv)),
                           ("g", g, (B, H, dk)), ("beta", beta, (B, H))):
        _check(t, name, shape, dt, dev)
    n_slots = S_pool.shape[0]
    _check(S_pool, "S_pool", (n_slots, H, dk, dv), torch.float32, dev)
    _check(slots, "slots", (B,), torch.int32, dev)
    if o is None:
        o = torch.empty((B, H, dv), dtype=dt, device=dev)
    else:
        _check(o, "o", (B, H, dv), dt, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_decode_step_paged(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_pool), n_slots,
                                         _ptr(slots), _ptr(o), B, H, dk, dv, DTYPE[dt], _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_decode_step_paged", rc)
    return o


def kda_state_compose(M, S, N=None, *, out=None, stream=None):
    """out = M @ S + N per head: M [..., dk, dk], S and N [..., dk, dv] fp32 CUDA tensors (N may be None).

    out may be S or N itself.  The leading dimensions are flattened into heads.
    """
    dk, dv = S.shape[-2], S.shape[-1]
    lead = tuple(S.shape[:-2])
    dev = S.device
    _check(M, "M", lead + (dk, dk), torch.float32, dev)
    if N is not None:
        _check(N, "N", lead + (dk, dv), torch.float32, dev)
    _check(S, "S", lead + (dk, dv), torch.float32, dev)
    if out is None:
        out = torch.empty_like(S)
    else:
        _check(out, "out", lead + (dk, dv), torch.float32, dev)
    count = 1
    for x in lead:
        count *= x
    with torch.cuda.device(dev):
        rc = lib().kda_state_compose(_ptr(M), _ptr(S), _ptr(N), _ptr(out), count, dk, dv, _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_state_compose", rc)
    return out


def kda_output_correct(C, S_in, o_in, *, out=None, stream=None):
    """out = o_in + per token S_in^T C: C [B, T, H, dk], o_in [B, T, H, dv] (same dtype) and S_in
    [B, H, dk, dv] fp32 CUDA tensors.  out may be o_in itself.  The output correction of a segment
    run from a zero state (context parallelism): C is the output of the same segment with v = 0 and
    S0 = I."""
    B, T, H, dk = C.shape
    dv = o_in.shape[-1]
    dev, dt = C.device, C.dtype
    if dt not in DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    _check(C, "C", (B, T, H, dk), dt, dev)
    _check(o_in, "o_in", (B, T, H, dv), dt, dev)
    _check(S_in, "S_in", (B, H, dk, dv), torch.float32, dev)
    if out is None:
        out = torch.empty_like(o_in)
    else:
        _check(out, "out", (B, T, H, dv), dt, dev)
    with torch.cuda.device(dev):
        rc = lib().kda_output_correct(_ptr(C), _ptr(S_in), _ptr(o_in), _ptr(out), B, T, H, dk, dv, DTYPE[dt],
                                      _stream_handle(stream))
    if rc != 0:
        raise KdaError("kda_output_correct", rc)
    return out


def kda_get_device_status(stream=None, device=None) -> int:
    """Synchronise the stream, then return and clear the device status word (0 = OK)."""
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(lib().kda_get_device_status(_stream_handle(stream)))


def kda_debug_set_wait_fault(mode: int, timeout_ns: int = 0) -> None:
    """Test hook: mode 1 makes tensor-core prefill launches time out a bounded device wait."""
    rc = lib().kda_debug_set_wait_fault(int(mode), int(timeout_ns))
    if rc != 0:
        raise KdaError("kda_debug_set_wait_fault", rc)
