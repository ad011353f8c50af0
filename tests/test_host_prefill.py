"""Prefill on host buffers (kda_forward_chunked_host).

The call cuts the work into segments of one batch entry and at most 2048 tokens, carries the
state between the segments of a sequence in device memory and overlaps copy-in, kernel and
copy-out.  Its outputs must be bitwise those of kda_forward_chunked on the same values: for one
segment and for several, with and without S0 / S_T, for both kernels, and for T = 0.  Argument
errors are reported before anything is enqueued (checked here without a GPU).
"""
import ctypes

import pytest
import torch

import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS

OK, INVALID, UNSUPPORTED, MISALIGNED = (STATUS[n] for n in
                                        ("KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                         "KDA_ERR_MISALIGNED"))

# ---------------------------------------------------------------------- C ABI checks (CPU)

BASE = 0x7F0000000000
SZ = 1 << 30


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrence_forward_b200 import build
    build.build()
    return kda.lib()


def ptrs():
    return [BASE + i * SZ for i in range(9)]   # q k v g beta S0 o S_T workspace


def host(L, p, B=2, T=1000, H=2, dk=128, dv=128, dtype=0, ws_bytes=None, impl=0):
    if ws_bytes is None:
        ws_bytes = L.kda_forward_chunked_host_workspace(T, H, dk, dv, dtype)
    return L.kda_forward_chunked_host(*p[:8], B, T, H, dk, dv, dtype, p[8], ws_bytes, impl, None)


def test_workspace_size(L):
    W = L.kda_forward_chunked_host_workspace
    state = 96 * 128 * 128 * 4
    assert W(0, 96, 128, 128, 0) == 2 * state                     # T = 0: the two state slots
    seg = 2048 * 96 * (3 * 128 + 2 * 128 + 1) * 2                 # q, k, g, v, o, beta of 2048 tokens
    assert W(8192, 96, 128, 128, 0) == 2 * seg + 2 * state
    assert W(65536, 96, 128, 128, 0) == W(8192, 96, 128, 128, 0)  # independent of T past one segment
    assert W(100, 2, 64, 64, 1) < W(100, 2, 128, 128, 1)
    assert W(100, 2, 96, 128, 0) == 0 and W(100, 0, 128, 128, 0) == 0 and W(-1, 2, 128, 128, 0) == 0
    assert W(100, 2, 128, 128, 7) == 0


def test_host_prefill_rejects_bad_arguments(L):
    assert host(L, ptrs(), B=0) == INVALID
    assert host(L, ptrs(), T=-1) == INVALID
    assert host(L, ptrs(), dk=96) == UNSUPPORTED
    assert host(L, ptrs(), dtype=5) == UNSUPPORTED
    assert host(L, ptrs(), impl=9) == INVALID
    p = ptrs(); p[8] = None
    assert host(L, p) == INVALID                                  # no workspace
    p = ptrs(); p[8] += 8
    assert host(L, p) == MISALIGNED
    assert host(L, ptrs(), ws_bytes=L.kda_forward_chunked_host_workspace(1000, 2, 128, 128, 0) - 1) == INVALID
    p = ptrs(); p[0] = None
    assert host(L, p) == INVALID                                  # missing input
    p = ptrs(); p[6] = p[0] + 4096
    assert host(L, p) == INVALID                                  # o inside q
    p = ptrs(); p[7] = p[6] + 64
    assert host(L, p) == INVALID                                  # S_T inside o
    p = ptrs(); p[7] = p[5] + 64
    assert host(L, p) == INVALID                                  # S_T partly over S0


# ---------------------------------------------------------------------- GPU

gpu = pytest.mark.gpu


def _inputs(B, T, H, d, dtype, seed, s0):
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    q, k, v, g, beta, S0 = make_prefill_inputs(B, T, H, d, d, dtype, seed=seed, s0_std=0.05, device="cuda")
    return q, k, v, g, beta, (S0 if s0 else None)


def _pinned(t):
    return None if t is None else t.to("cpu").pin_memory()


@gpu
@pytest.mark.parametrize("B,T,H,d,dtype,impl,s0", [
    (2, 5000, 3, 128, "bf16", "tcgen05", True),     # three segments per sequence, ragged last one
    (3, 2048, 2, 128, "bf16", "tcgen05", False),    # exactly one segment, zero initial state
    (4, 5000, 2, 128, "bf16", "tcgen05", True),     # state slot b % 2 reused by b + 2, each with an S0 copy-in
    (1, 4097, 2, 128, "bf16", "auto", True),        # one token past two segments
    (2, 300, 2, 64, "fp32", "simt", True),          # the CUDA-core kernel
    (2, 4200, 1, 64, "bf16", "simt", False),
    (2, 4200, 2, 64, "bf16", "tcgen05", True),      # head size 64 on the tensor-core kernel
])
def test_host_prefill_equals_device_prefill_bitwise(B, T, H, d, dtype, impl, s0):
    q, k, v, g, beta, S0 = _inputs(B, T, H, d, dtype, seed=3, s0=s0)
    o_ref, ST_ref = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl=impl)
    hq, hk, hv, hg, hb = (_pinned(x) for x in (q, k, v, g, beta))
    hS0 = _pinned(S0)
    o, ST = kda.kda_forward_chunked_host(hq, hk, hv, hg, hb, hS0, impl=impl)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    assert torch.equal(o, o_ref.cpu()) and torch.equal(ST, ST_ref.cpu())
    assert hS0 is None or torch.equal(hS0, S0.cpu())            # the input state is left alone


@gpu
def test_host_prefill_in_place_state_pageable_inputs_and_no_final_state():
    q, k, v, g, beta, S0 = _inputs(2, 2500, 2, 128, "bf16", seed=5, s0=True)
    o_ref, ST_ref = kda.kda_forward_chunked(q, k, v, g, beta, S0)
    cq, ck, cv, cg, cb = (x.cpu() for x in (q, k, v, g, beta))   # pageable: staged copies
    S = S0.cpu()
    o, ST = kda.kda_forward_chunked_host(cq, ck, cv, cg, cb, S, S_T=S)
    torch.cuda.synchronize()
    assert ST is S and torch.equal(S, ST_ref.cpu()) and torch.equal(o, o_ref.cpu())
    o2, ST2 = kda.kda_forward_chunked_host(cq, ck, cv, cg, cb, S0.cpu(), return_state=False)
    torch.cuda.synchronize()
    assert ST2 is None and torch.equal(o2, o_ref.cpu())


@gpu
def test_host_prefill_with_no_tokens_copies_the_state():
    S0 = torch.randn((2, 3, 128, 128)).pin_memory()
    z = torch.empty((2, 0, 3, 128), dtype=torch.bfloat16).pin_memory()
    zb = torch.empty((2, 0, 3), dtype=torch.bfloat16).pin_memory()
    o, ST = kda.kda_forward_chunked_host(z, z, z, z, zb, S0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 3, 128) and torch.equal(ST, S0)
    o, ST = kda.kda_forward_chunked_host(z, z, z, z, zb, None)
    torch.cuda.synchronize()
    assert torch.equal(ST, torch.zeros_like(S0))


@gpu
def test_host_prefill_reuses_a_given_workspace_and_rejects_a_small_one():
    q, k, v, g, beta, S0 = _inputs(1, 3000, 2, 128, "bf16", seed=7, s0=True)
    o_ref, ST_ref = kda.kda_forward_chunked(q, k, v, g, beta, S0)
    args = [_pinned(x) for x in (q, k, v, g, beta, S0)]
    ws = torch.empty(kda.host_workspace_bytes(3000, 2), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        o, ST = kda.kda_forward_chunked_host(*args, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref.cpu()) and torch.equal(ST, ST_ref.cpu())
    with pytest.raises(kda.KdaError) as err:
        kda.kda_forward_chunked_host(*args, workspace=ws[:-16])
    assert err.value.status == INVALID
