"""The C ABI: the library loads, exports what include/kda.h declares, and rejects bad
arguments on the host before touching the GPU (these run without a GPU)."""
import ctypes
import os
import re

import pytest

import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED, MISALIGNED = (STATUS[n] for n in
                                        ("KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                         "KDA_ERR_MISALIGNED"))


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrence_forward_b200 import build
    build.build()
    return kda.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("kda_forward_chunked", "kda_forward_chunked_impl", "kda_decode_step",
                 "kda_get_device_status", "kda_status_string", "kda_version"):
        assert name in syms


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), f"{name} declared in include/kda.h but not exported"


def test_status_strings(L):
    for name, code in STATUS.items():
        assert kda.kda_status_string(code) == name
    assert kda.kda_status_string(12345) == "KDA_ERR_UNKNOWN"
    assert L.kda_version() >= 100


# Fake, never-dereferenced device addresses: the host checks only do arithmetic on them.
BASE = 0x7F0000000000
SZ = 1 << 30


def ptrs(n=8, misalign=None):
    out = [BASE + i * SZ for i in range(n)]
    if misalign is not None:
        out[misalign] += 8
    return out


def fwd(L, p, B=1, T=64, H=2, dk=128, dv=128, dtype=0, impl=0):
    q, k, v, g, beta, S0, o, ST = p
    return L.kda_forward_chunked_impl(q, k, v, g, beta, S0, o, ST, B, T, H, dk, dv, dtype, impl, None)


def dec(L, p, B=2, H=3, dk=128, dv=128, dtype=0):
    q, k, v, g, beta, S, o = p[:7]
    return L.kda_decode_step(q, k, v, g, beta, S, o, B, H, dk, dv, dtype, None)


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(T=-1), dict(B=-3)])
def test_forward_rejects_bad_sizes(L, kw):
    assert fwd(L, ptrs(), **kw) == INVALID


@pytest.mark.parametrize("kw", [dict(dk=96), dict(dv=32), dict(dk=256), dict(dtype=7)])
def test_forward_rejects_unsupported(L, kw):
    assert fwd(L, ptrs(), **kw) == UNSUPPORTED


@pytest.mark.parametrize("which", range(8))
def test_forward_rejects_misaligned(L, which):
    assert fwd(L, ptrs(misalign=which)) == MISALIGNED


@pytest.mark.parametrize("which", range(6))
def test_forward_rejects_null_required_pointer(L, which):
    p = ptrs()
    idx = [0, 1, 2, 3, 4, 6][which]  # q k v g beta o
    p[idx] = None
    assert fwd(L, p) == INVALID


def test_forward_rejects_output_overlapping_input(L):
    p = ptrs()
    p[6] = p[0] + 4096           # o inside q
    assert fwd(L, p) == INVALID
    p = ptrs()
    p[7] = p[5] + 4096           # S_T partially overlapping S0 (exact aliasing is allowed)
    assert fwd(L, p) == INVALID
    p = ptrs()
    p[7] = p[2]                  # S_T on top of v
    assert fwd(L, p) == INVALID


def test_forward_rejects_bad_impl(L):
    assert fwd(L, ptrs(), impl=9) == INVALID


def test_forward_tcgen05_rejects_shapes_it_does_not_cover(L):
    # the tensor-core kernel covers bf16 only (head sizes 64 and 128, like every kernel)
    assert fwd(L, ptrs(), dtype=1, impl=1) == UNSUPPORTED
    for dk, dv in ((64, 64), (128, 64), (64, 128)):
        assert fwd(L, ptrs(), dk=dk, dv=dv, dtype=1, impl=1) == UNSUPPORTED
        assert fwd(L, ptrs(), dk=dk, dv=dv, dtype=1, impl=1, T=0) == UNSUPPORTED


def test_decode_rejects_bad_arguments(L):
    assert dec(L, ptrs(), B=0) == INVALID
    assert dec(L, ptrs(), dk=80) == UNSUPPORTED
    assert dec(L, ptrs(), dtype=3) == UNSUPPORTED
    for i in range(7):
        assert dec(L, ptrs(misalign=i)) == MISALIGNED
    p = ptrs()
    p[5] = None                  # S must be given
    assert dec(L, p) == INVALID
    p = ptrs()
    p[6] = p[5] + 1024           # o inside S
    assert dec(L, p) == INVALID


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    mod = importlib.reload(kda)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mod, "_lib", None)
    with pytest.raises(ImportError):
        mod.lib()
    importlib.reload(kda)


def test_wait_fault_hook_validates_arguments(L):
    assert L.kda_debug_set_wait_fault(2, 10_000_000) == INVALID
    assert L.kda_debug_set_wait_fault(1, 10) == INVALID            # below 1 ms
    assert L.kda_debug_set_wait_fault(1, 20_000_000_000) == INVALID  # above 10 s
    assert L.kda_debug_set_wait_fault(1, 20_000_000) == OK
    assert L.kda_debug_set_wait_fault(0, 0) == OK
