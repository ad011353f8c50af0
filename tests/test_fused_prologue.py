"""The prologue-fused prefill: g = -5 sigmoid(z_g), beta = sigmoid(z_beta), q and k L2-normalised,
all inside the kernels' load stage.

CPU: the oracle's prologue pinned to values the definition fixes (sigmoid(0) = 1/2, the limits of
the gate, unit rows, invariance to the scale of q and k, the single-token closed form with
parallel q and k).  GPU: both prefill kernels against the oracle, bitwise invariance to
power-of-two scalings of q and k, exact zeros for a zero query row.
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_forward_b200 as kda
from helpers import max_rel_err


def raw_problem(rng, B, T, H, dk, dv, zg_scale=1.0):
    q = rng.standard_normal((B, T, H, dk)) * 3.0
    k = rng.standard_normal((B, T, H, dk)) * 0.5
    v = rng.standard_normal((B, T, H, dv))
    z_g = rng.standard_normal((B, T, H, dk)) * zg_scale
    z_b = rng.standard_normal((B, T, H))
    return q, k, v, z_g, z_b


def test_prologue_values():
    z = np.array([0.0, 40.0, -40.0, 2.0])
    q, k, g, beta = oracle.prologue(np.ones((1, 1, 1, 4)), np.ones((1, 1, 1, 4)), z.reshape(1, 1, 1, 4),
                                    np.zeros((1, 1, 1)))
    assert g[0, 0, 0, 0] == -2.5
    assert abs(g[0, 0, 0, 1] + 5.0) < 1e-15 and abs(g[0, 0, 0, 2]) < 1e-15
    assert abs(g[0, 0, 0, 3] + 5.0 / (1.0 + np.exp(-2.0))) < 1e-15
    assert beta[0, 0, 0] == 0.5
    assert np.allclose(q, 0.5) and np.allclose(k, 0.5)       # unit rows
    qz, _, _, _ = oracle.prologue(np.zeros((1, 1, 1, 4)), np.ones((1, 1, 1, 4)), np.zeros((1, 1, 1, 4)),
                                  np.zeros((1, 1, 1)))
    assert np.all(qz == 0.0)                                  # a zero row stays zero


def test_fused_oracle_is_invariant_to_the_scale_of_q_and_k():
    rng = np.random.default_rng(3)
    q, k, v, z_g, z_b = raw_problem(rng, 1, 40, 2, 8, 6)
    o1, S1 = oracle.forward_fused(q, k, v, z_g, z_b)
    o2, S2 = oracle.forward_fused(q * 7.5, k * 0.01, v, z_g, z_b)
    assert max_rel_err(o2, o1) < 1e-13 and max_rel_err(S2, S1) < 1e-13


def test_single_token_with_parallel_query_and_key():
    """o_1 = beta (q.k) v with unit q = k: o_1 = sigmoid(z_beta) v, whatever the gate."""
    rng = np.random.default_rng(4)
    k = rng.standard_normal((1, 1, 1, 8))
    v = rng.standard_normal((1, 1, 1, 5))
    z_b = np.array([[[0.7]]])
    o, _ = oracle.forward_fused(k * 3.0, k, v, rng.standard_normal((1, 1, 1, 8)), z_b)
    assert np.allclose(o[0, 0, 0], v[0, 0, 0] / (1.0 + np.exp(-0.7)), rtol=0, atol=1e-14)


# ---------------------------------------------------------------------- GPU

def gpu_raw(B, T, H, d, dtype, seed, zg_mean=0.0):
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_raw_inputs
    return make_prefill_raw_inputs(B, T, H, d, d, dtype, seed=seed, s0_std=0.05, zg_mean=zg_mean, device="cuda")


CASES = [("bf16", "tcgen05", 128, 1, 1000, 4), ("bf16", "tcgen05", 64, 2, 300, 3), ("bf16", "simt", 128, 2, 300, 2), ("fp32", "simt", 64, 1, 256, 3),
         ("fp32", "simt", 128, 1, 130, 2)]


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,impl,d,B,T,H", CASES)
def test_fused_prefill_matches_the_oracle(dtype, impl, d, B, T, H):
    q, k, v, z_g, z_b, S0 = gpu_raw(B, T, H, d, dtype, seed=1)
    o, ST = kda.kda_forward_chunked_fused(q, k, v, z_g, z_b, S0, impl=impl)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref = oracle.forward_fused(q, k, v, z_g, z_b, S0)
    tol = 2e-2 if dtype == "bf16" else 1e-4
    eo = max_rel_err(o.double().cpu().numpy(), o_ref)
    es = max_rel_err(ST.double().cpu().numpy(), ST_ref)
    assert eo <= tol and es <= tol, (eo, es)


@pytest.mark.gpu
@pytest.mark.parametrize("impl", ["tcgen05", "simt"])
def test_fused_prefill_is_invariant_to_power_of_two_scalings(impl):
    q, k, v, z_g, z_b, S0 = gpu_raw(2, 200, 2, 128, "bf16", seed=2)
    o1, S1 = kda.kda_forward_chunked_fused(q, k, v, z_g, z_b, S0, impl=impl)
    o2, S2 = kda.kda_forward_chunked_fused((q * 2).contiguous(), (k * 0.25).contiguous(), v, z_g, z_b, S0, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.gpu
@pytest.mark.parametrize("impl", ["tcgen05", "simt"])
def test_zero_query_rows_give_zero_outputs(impl):
    q, k, v, z_g, z_b, S0 = gpu_raw(1, 130, 2, 128, "bf16", seed=3)
    q[:, 5] = 0
    q[:, 77, 1] = 0
    o, _ = kda.kda_forward_chunked_fused(q, k, v, z_g, z_b, S0, impl=impl)
    torch.cuda.synchronize()
    assert bool((o[:, 5] == 0).all()) and bool((o[:, 77, 1] == 0).all())
    assert not bool((o[:, 6] == 0).all())


@pytest.mark.gpu
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 128, 129, 200])
def test_fused_prefill_chunk_counts(T, d):
    """The tensor-core kernel's prologue converts the gate of chunks 0 and 1 before its loop and of
    chunk c + 2 inside it, and loads the next gate after each conversion: one, two and three chunks
    (and ragged tails) take different paths through that pipeline."""
    q, k, v, z_g, z_b, S0 = gpu_raw(2, T, 2, d, "bf16", seed=T)
    o, ST = kda.kda_forward_chunked_fused(q, k, v, z_g, z_b, S0, impl="tcgen05")
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref = oracle.forward_fused(q, k, v, z_g, z_b, S0)
    eo = max_rel_err(o.double().cpu().numpy(), o_ref)
    es = max_rel_err(ST.double().cpu().numpy(), ST_ref)
    assert eo <= 2e-2 and es <= 2e-2, (eo, es)
