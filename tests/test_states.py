"""Intermediate states every `interval` tokens (the prefix-cache boundaries).

The state after token n*interval must be the state a run over the first n*interval tokens
ends in (split/resume consistency: the recurrence is a left fold over tokens, so a prefix's
final state is the full run's state at that token).

CPU: the oracle's state output against its own prefix runs, and the C ABI's argument checks.
GPU: both prefill kernels against the oracle, bitwise against their own prefix runs, and
o / S_T unchanged by the extra output.
"""
import numpy as np
import pytest

import oracle
import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS
from helpers import max_rel_err, random_problem

OK, INVALID, UNSUPPORTED, MISALIGNED = (STATUS[n] for n in
                                        ("KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                         "KDA_ERR_MISALIGNED"))


# ---------------------------------------------------------------------- oracle (CPU)

@pytest.mark.parametrize("T,interval", [(200, 64), (256, 64), (130, 128), (50, 64)])
def test_oracle_states_are_prefix_final_states(T, interval):
    rng = np.random.default_rng(5)
    q, k, v, g, beta, S0 = random_problem(rng, 2, T, 3, 8, 6)
    o, ST, S_mid = oracle.forward_states(q, k, v, g, beta, S0, interval=interval)
    o_full, ST_full = oracle.forward(q, k, v, g, beta, S0)
    assert S_mid.shape == (2, 3, T // interval, 8, 6)
    assert np.array_equal(o, o_full) and np.array_equal(ST, ST_full)
    for n in range(T // interval):
        e = (n + 1) * interval
        _, ST_pre = oracle.forward(q[:, :e], k[:, :e], v[:, :e], g[:, :e], beta[:, :e], S0)
        assert np.array_equal(S_mid[:, :, n], ST_pre)


def test_oracle_states_resume():
    """Resuming from a recorded state reproduces the rest of the run (I7)."""
    rng = np.random.default_rng(6)
    q, k, v, g, beta, S0 = random_problem(rng, 1, 192, 2, 8, 8)
    o, ST, S_mid = oracle.forward_states(q, k, v, g, beta, S0, interval=64)
    o2, ST2 = oracle.forward(q[:, 128:], k[:, 128:], v[:, 128:], g[:, 128:], beta[:, 128:], S_mid[:, :, 1])
    assert max_rel_err(o2, o[:, 128:]) < 1e-13 and max_rel_err(ST2, ST) < 1e-13


# ---------------------------------------------------------------------- C ABI checks (CPU)

BASE = 0x7F0000000000
SZ = 1 << 30


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrence_forward_b200 import build
    build.build()
    return kda.lib()


def call(L, S_mid, interval, T=1024, B=1, H=2, dk=128, dv=128, dtype=0, impl=0, misalign=None):
    p = [BASE + i * SZ for i in range(8)]
    if misalign is not None:
        p[misalign] += 8
    q, k, v, g, beta, S0, o, ST = p
    return L.kda_forward_chunked_states(q, k, v, g, beta, S0, o, ST, S_mid, interval, B, T, H, dk, dv,
                                        dtype, impl, None)


def test_states_rejects_bad_interval(L):
    good = BASE + 9 * SZ
    assert call(L, good, 0) == INVALID
    assert call(L, good, -512) == INVALID
    assert call(L, good, 100) == UNSUPPORTED
    assert call(L, good, 32) == UNSUPPORTED


def test_states_requires_the_output_when_a_boundary_falls_inside(L):
    assert call(L, None, 512) == INVALID          # T = 1024: two states to write
    assert call(L, BASE + 9 * SZ + 8, 512) == MISALIGNED


def test_states_rejects_overlap(L):
    assert call(L, BASE + 6 * SZ + 4096, 512) == INVALID   # inside o
    assert call(L, BASE + 5 * SZ, 512) == INVALID          # on S0
    assert call(L, BASE + 7 * SZ - 4096, 512) == INVALID   # runs into S_T
    assert call(L, BASE + 0 * SZ, 512) == INVALID          # on q


def test_states_still_checks_the_prefill_arguments(L):
    good = BASE + 9 * SZ
    assert call(L, good, 512, misalign=2) == MISALIGNED
    assert call(L, good, 512, dk=96) == UNSUPPORTED
    assert call(L, good, 512, B=0) == INVALID
    assert call(L, good, 512, impl=7) == INVALID


# ---------------------------------------------------------------------- GPU

gpu = pytest.mark.gpu
TOL = {"bf16": 2e-2, "fp32": 1e-4}


def _torch():
    import torch
    return torch


def to_np(t):
    torch = _torch()
    return t.detach().to("cpu", torch.float64).numpy()


def gpu_case(B, T, H, dk, dv, dtype, seed=0):
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    return make_prefill_inputs(B, T, H, dk, dv, dtype, seed=seed, s0_std=0.05, zg_mean=-1.0, device="cuda")


CASES = [  # (B, T, H, dk, dv, dtype, impl, interval)
    (2, 1100, 3, 128, 128, "bf16", "auto", 512),
    (1, 700, 2, 128, 128, "bf16", "tcgen05", 64),
    (1, 1024, 2, 128, 128, "bf16", "tcgen05", 256),
    (1, 700, 2, 64, 128, "bf16", "tcgen05", 128),     # head size 64 embedded in the 128-wide tiles
    (2, 600, 2, 128, 64, "bf16", "tcgen05", 64),
    (2, 300, 2, 64, 128, "fp32", "simt", 64),
    (1, 520, 2, 128, 128, "bf16", "simt", 128),
]


@gpu
@pytest.mark.parametrize("B,T,H,dk,dv,dtype,impl,interval", CASES)
def test_states_match_oracle(B, T, H, dk, dv, dtype, impl, interval):
    torch = _torch()
    q, k, v, g, beta, S0 = gpu_case(B, T, H, dk, dv, dtype)
    o, ST, S_mid = kda.kda_forward_chunked_states(q, k, v, g, beta, S0, interval=interval, impl=impl)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref, S_mid_ref = oracle.forward_states(q, k, v, g, beta, S0, interval=interval)
    assert S_mid.shape == (B, H, T // interval, dk, dv)
    for n in range(T // interval):
        e = max_rel_err(to_np(S_mid[:, :, n]), S_mid_ref[:, :, n])
        assert e <= TOL[dtype], (n, e)
    assert max_rel_err(to_np(o), o_ref) <= TOL[dtype]
    assert max_rel_err(to_np(ST), ST_ref) <= TOL[dtype]


@gpu
@pytest.mark.parametrize("impl", ["tcgen05", "simt"])
def test_states_are_bitwise_prefix_states_and_leave_outputs_unchanged(impl):
    torch = _torch()
    B, T, H, interval = 1, 1000, 3, 256
    q, k, v, g, beta, S0 = gpu_case(B, T, H, 128, 128, "bf16", seed=4)
    o, ST, S_mid = kda.kda_forward_chunked_states(q, k, v, g, beta, S0, interval=interval, impl=impl)
    o_plain, ST_plain = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(o, o_plain) and torch.equal(ST, ST_plain)
    for n in range(T // interval):
        e = (n + 1) * interval
        args = [x[:, :e].contiguous() for x in (q, k, v, g, beta)]
        _, ST_pre = kda.kda_forward_chunked(*args, S0, impl=impl)
        torch.cuda.synchronize()
        assert torch.equal(S_mid[:, :, n], ST_pre), n
    assert kda.kda_get_device_status() == 0


@gpu
def test_states_interval_longer_than_the_sequence():
    torch = _torch()
    q, k, v, g, beta, S0 = gpu_case(1, 300, 2, 128, 128, "bf16", seed=2)
    o, ST, S_mid = kda.kda_forward_chunked_states(q, k, v, g, beta, S0, interval=512)
    o_plain, ST_plain = kda.kda_forward_chunked(q, k, v, g, beta, S0)
    torch.cuda.synchronize()
    assert S_mid.shape == (1, 2, 0, 128, 128)
    assert torch.equal(o, o_plain) and torch.equal(ST, ST_plain)


@gpu
def test_states_resume_from_a_boundary_on_the_gpu():
    """Prefix cache use: resume from S_mid at token 512 and finish the sequence."""
    torch = _torch()
    q, k, v, g, beta, S0 = gpu_case(2, 1536, 2, 128, 128, "bf16", seed=8)
    o, ST, S_mid = kda.kda_forward_chunked_states(q, k, v, g, beta, S0, interval=512)
    rest = [x[:, 512:].contiguous() for x in (q, k, v, g, beta)]
    o2, ST2 = kda.kda_forward_chunked(*rest, S_mid[:, :, 0].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(o2, o[:, 512:]) and torch.equal(ST2, ST)
