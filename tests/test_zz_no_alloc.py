"""kda_forward_chunked_host_noalloc: the host-buffer prefill for callers that cannot allocate device memory.

Who calls it: a program that holds only host arrays and reaches the library through a plain C
foreign-function interface, with no CUDA allocator of its own to make the device workspace that
kda_forward_chunked_host needs; or an engine whose device memory is all owned by a pool that
allows no allocation outside it (where a cudaMalloc would also stall the device mid-work).  The
entry point stages everything through one fixed scratch array the library reserves per device when
it is loaded (KDA_NOALLOC_SCRATCH_BYTES), so such a caller passes host buffers and a stream only.

The GPU test calls it through the C ABI (ctypes, no Python wrapper in between) twice in a row on
different problems and compares each result with the workspace-based kda_forward_chunked_host on the
same inputs, within the parity tolerance used throughout the tests (2e-2 bf16, 1e-4 fp32); by
construction the two are also bitwise equal.  The second call starts from a zero state after the
first left its own state in the shared scratch, so a stale value would show.  The CPU tests check
the size limit and the argument checks, which return before anything touches a GPU.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS, DTYPE, IMPL
from helpers import max_rel_err

OK, INVALID, UNSUPPORTED = STATUS["KDA_OK"], STATUS["KDA_ERR_INVALID_ARG"], STATUS["KDA_ERR_UNSUPPORTED"]
SCRATCH_BYTES = 32 << 20      # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrence_forward_b200 import build
    build.build()
    return kda.lib()


# ---------------------------------------------------------------------- argument and size checks (CPU)

BASE = 0x7F0000000000
SZ = 1 << 34


def noalloc(L, p, B=1, T=100, H=4, dk=128, dv=128, dtype=0, impl=0):
    # fake host addresses: the checks below all return before any byte is touched
    return L.kda_forward_chunked_host_noalloc(*p, B, T, H, dk, dv, dtype, impl, None)


def fake_ptrs():
    return [BASE + i * SZ for i in range(8)]   # q k v g beta S0 o S_T


def test_declared_scratch_size_matches_the_header():
    import re
    import os
    header = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "kda.h")
    m = re.search(r"#define\s+KDA_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", open(header).read())
    assert m and int(m.group(1)) << int(m.group(2)) == SCRATCH_BYTES


def test_problems_beyond_the_scratch_are_refused(L):
    # one batch entry's state plus 64 tokens of every input and output must fit: H <= 227 at bf16
    # d = 128, H <= 146 at fp32 d = 128; the state alone decides for T = 0
    assert noalloc(L, fake_ptrs(), H=228) == UNSUPPORTED
    assert noalloc(L, fake_ptrs(), H=228, T=5000) == UNSUPPORTED
    assert noalloc(L, fake_ptrs(), H=147, dtype=1) == UNSUPPORTED
    assert noalloc(L, fake_ptrs(), H=513, T=0) == UNSUPPORTED


def test_bad_arguments_are_refused_before_anything_runs(L):
    assert noalloc(L, fake_ptrs(), B=0) == INVALID
    assert noalloc(L, fake_ptrs(), T=-1) == INVALID
    assert noalloc(L, fake_ptrs(), impl=9) == INVALID
    assert noalloc(L, fake_ptrs(), dk=96) == UNSUPPORTED
    assert noalloc(L, fake_ptrs(), dk=64, dv=64, dtype=1, impl=IMPL["tcgen05"]) == UNSUPPORTED   # fp32 has no tensor-core kernel
    assert noalloc(L, fake_ptrs(), dtype=1, impl=IMPL["tcgen05"]) == UNSUPPORTED
    p = fake_ptrs(); p[0] = None
    assert noalloc(L, p) == INVALID
    p = fake_ptrs(); p[6] = p[0] + 4096
    assert noalloc(L, p) == INVALID                                # o inside q
    p = fake_ptrs(); p[7] = p[5] + 64
    assert noalloc(L, p) == INVALID                                # S_T partly over S0


# ---------------------------------------------------------------------- GPU


def _problem(B, T, H, d, dtype, seed, s0):
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    q, k, v, g, beta, S0 = make_prefill_inputs(B, T, H, d, d, dtype, seed=seed, s0_std=0.05, device="cpu")
    pin = lambda x: None if x is None else x.contiguous().pin_memory()
    return [pin(x) for x in (q, k, v, g, beta)] + [pin(S0) if s0 else None]


def _call_noalloc(L, q, k, v, g, beta, S0, impl):
    """One call through the C ABI on the current stream; returns (o, S_T) as host tensors."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty((B, T, H, dv), dtype=q.dtype).pin_memory()
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32).pin_memory()
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = torch.cuda.current_stream()
    rc = L.kda_forward_chunked_host_noalloc(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(S0), ptr(o), ptr(ST),
                                            B, T, H, dk, dv, DTYPE[q.dtype], IMPL[impl],
                                            ctypes.c_void_p(stream.cuda_stream) if stream.cuda_stream else None)
    assert rc == OK, kda.kda_status_string(rc)
    stream.synchronize()
    return o, ST


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,H,d,dtype,impl", [
    (2, 1000, 96, 128, "bf16", "auto"),    # 192-token segments: five full and a 40-token tail per sequence
    (1, 600, 96, 64, "fp32", "auto"),      # 256-token segments on the fp32 kernel
])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row(L, B, T, H, d, dtype, impl):
    torch.cuda.init()
    for call, (seed, s0) in enumerate(((11, True), (12, False))):
        q, k, v, g, beta, S0 = _problem(B, T, H, d, dtype, seed, s0)
        o, ST = _call_noalloc(L, q, k, v, g, beta, S0, impl)
        o_ref, ST_ref = kda.kda_forward_chunked_host(q, k, v, g, beta, S0, impl=impl)
        torch.cuda.synchronize()
        assert kda.kda_get_device_status() == 0
        tol = TOL[q.dtype]
        assert max_rel_err(o.double().numpy(), o_ref.double().numpy()) <= tol, call
        assert max_rel_err(ST.double().numpy(), ST_ref.double().numpy()) <= tol, call
        assert torch.equal(o, o_ref) and torch.equal(ST, ST_ref), call
        if S0 is not None:
            assert torch.equal(S0, _problem(B, T, H, d, dtype, seed, s0)[5])   # the input state is left alone
