"""CUDA path vs the fp64 oracle, element by element, on the same seeded inputs (GPU).

Tolerance (the stated bar): max |x - ref| / max |ref| per output tensor <= 2e-2 for bf16
inputs and <= 1e-4 for fp32 inputs.  Exact-zero and exact-recall cases are checked exactly
(up to the output's own rounding).
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs, make_decode_inputs
from helpers import max_rel_err, check_parity

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "fp32": 1e-4}
DEV = "cuda"


def to_np(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def run_prefill(inputs, impl="auto"):
    q, k, v, g, beta, S0 = inputs
    o, ST = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl=impl)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    return o, ST


def check_prefill(inputs, dtype, impl="auto"):
    o, ST = run_prefill(inputs, impl)
    o_ref, ST_ref = oracle.forward(*inputs)
    B, T, H, dk = inputs[0].shape
    case = f"{impl} {dtype} B{B} T{T} H{H} dk{dk} dv{inputs[2].shape[-1]}{' S0' if inputs[5] is not None else ''}"
    eo = check_parity(case, "o", to_np(o), o_ref, TOL[dtype], (0, 2))["rel"]
    es = check_parity(case, "S_T", to_np(ST), ST_ref, TOL[dtype], (0, 1))["rel"]
    return eo, es


def gpu_inputs(B, T, H, dk, dv, dtype, s0_std=0.0, zg_mean=0.0, seed=0):
    return make_prefill_inputs(B, T, H, dk, dv, dtype, seed=seed, s0_std=s0_std, zg_mean=zg_mean,
                               device=DEV)


IMPLS = ["simt", "auto"]


# ---------------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_decode_matches_oracle(dtype, dk, dv):
    B, H, steps = 5, 7, 6
    gen = torch.Generator(device=DEV)
    gen.manual_seed(3)
    S = (torch.randn((B, H, dk, dv), generator=gen, device=DEV) * 0.1).contiguous()
    S_ref = to_np(S).copy()
    for _ in range(steps):
        q, k, v, g, beta = make_decode_inputs(B, H, dk, dv, dtype, gen=gen, device=DEV)
        o = kda.kda_decode_step(q, k, v, g, beta, S)
        o_ref = oracle.decode_step(q, k, v, g, beta, S_ref)
        torch.cuda.synchronize()
        assert max_rel_err(to_np(o), o_ref) <= TOL[dtype]
    assert max_rel_err(to_np(S), S_ref) <= TOL[dtype]
    assert kda.kda_get_device_status() == 0


def test_decode_equals_prefill_on_gpu():
    B, T, H, d = 2, 40, 3, 128
    q, k, v, g, beta, S0 = gpu_inputs(B, T, H, d, d, "bf16", s0_std=0.05, seed=11)
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0)
    S = S0.clone()
    outs = []
    for t in range(T):
        outs.append(kda.kda_decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                                        g[:, t].contiguous(), beta[:, t].contiguous(), S))
    o = torch.stack(outs, dim=1)
    torch.cuda.synchronize()
    assert max_rel_err(to_np(o), o_ref) <= 2e-2
    assert max_rel_err(to_np(S), ST_ref) <= 2e-2


# ---------------------------------------------------------------------- prefill, small

@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_small_fp32_config(impl):
    """The fp32 workload (B1 T256 H2 d64, S0 = 0) in full at 1e-4."""
    check_prefill(gpu_inputs(1, 256, 2, 64, 64, "fp32"), "fp32", impl)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_prefill_shapes(impl, dtype, dk, dv, T):
    # AUTO: bf16 on the tensor-core kernel (head size 64 embedded in its 128-wide tiles), fp32 on
    # the CUDA-core kernel
    inputs = gpu_inputs(2, T, 3, dk, dv, dtype, s0_std=0.05, seed=T)
    check_prefill(inputs, dtype, impl)


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_zero_length_copies_state(impl):
    q, k, v, g, beta, S0 = gpu_inputs(2, 0, 3, 128, 128, "bf16", s0_std=0.1)
    o, ST = run_prefill((q, k, v, g, beta, S0), impl)
    assert o.shape == (2, 0, 3, 128)
    assert torch.equal(ST, S0)
    o, ST = run_prefill((q, k, v, g, beta, None), impl)
    assert torch.count_nonzero(ST) == 0


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_beta_zero_gives_exact_zero(impl):
    q, k, v, g, beta, _ = gpu_inputs(1, 130, 4, 128, 128, "bf16")
    o, ST = run_prefill((q, k, v, g, torch.zeros_like(beta), None), impl)
    assert torch.count_nonzero(o) == 0 and torch.count_nonzero(ST) == 0


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_orthonormal_recall(impl):
    """g = 0, beta = 1, permuted standard-basis keys: querying with k_i returns v_i."""
    d, n = 128, 100
    gen = torch.Generator().manual_seed(5)
    perm = torch.randperm(d, generator=gen)[:n]
    keys = torch.eye(d)[perm]
    vals = torch.randn((n, d), generator=gen)
    T = 2 * n
    q = torch.zeros((1, T, 1, d)); k = torch.zeros((1, T, 1, d)); v = torch.zeros((1, T, 1, d))
    beta = torch.zeros((1, T, 1))
    k[0, :n, 0] = keys; v[0, :n, 0] = vals; beta[0, :n, 0] = 1.0
    order = torch.randperm(n, generator=gen)
    q[0, n:, 0] = keys[order]
    k[0, n:, 0] = torch.eye(d)[0]
    inputs = tuple(x.to(DEV, torch.bfloat16).contiguous() for x in (q, k, v, torch.zeros_like(q), beta)) + (None,)
    o, _ = run_prefill(inputs, impl)
    expect = vals[order].to(torch.bfloat16).float()
    got = o[0, n:, 0].float().cpu()
    assert torch.max(torch.abs(got - expect)) <= 2e-2 * torch.max(torch.abs(expect))


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_split_resume_and_in_place_state(impl):
    B, T, H, d = 1, 300, 2, 128
    q, k, v, g, beta, S0 = gpu_inputs(B, T, H, d, d, "bf16", s0_std=0.05, seed=4)
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0)
    for T1 in (64, 100, 256):
        S = S0.clone()
        oa, _ = kda.kda_forward_chunked(q[:, :T1].contiguous(), k[:, :T1].contiguous(), v[:, :T1].contiguous(),
                                        g[:, :T1].contiguous(), beta[:, :T1].contiguous(), S, S_T=S, impl=impl)
        ob, _ = kda.kda_forward_chunked(q[:, T1:].contiguous(), k[:, T1:].contiguous(), v[:, T1:].contiguous(),
                                        g[:, T1:].contiguous(), beta[:, T1:].contiguous(), S, S_T=S, impl=impl)
        torch.cuda.synchronize()
        assert max_rel_err(to_np(torch.cat([oa, ob], dim=1)), o_ref) <= 2e-2
        assert max_rel_err(to_np(S), ST_ref) <= 2e-2


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_padding_tokens_are_no_ops(impl):
    B, T, H, d = 1, 100, 2, 128
    q, k, v, g, beta, S0 = gpu_inputs(B, T, H, d, d, "bf16", s0_std=0.05, seed=9)
    _, ST = run_prefill((q, k, v, g, beta, S0), impl)
    pad = 28
    z = lambda x: torch.cat([x, torch.zeros((B, pad) + x.shape[2:], dtype=x.dtype, device=DEV)], 1).contiguous()
    qp, kp, vp = z(q), z(k), z(v)
    kp[:, T:] = k[:, :pad]                 # nonzero keys, but beta = 0 and g = 0
    _, ST2 = run_prefill((qp, kp, vp, z(g), z(beta), S0), impl)
    assert torch.equal(ST, ST2) or max_rel_err(to_np(ST2), to_np(ST)) < 1e-6


# ---------------------------------------------------------------------- head size 64 on the tensor core

@pytest.mark.parametrize("dk,dv,B,T,H", [(64, 64, 2, 1000, 5), (64, 128, 1, 777, 3), (128, 64, 1, 777, 3)])
def test_prefill_head64_tensor_core_matches_oracle(dk, dv, B, T, H):
    """bf16 head size 64 on the chunkwise tensor-core kernel: several chunks and a ragged tail."""
    check_prefill(gpu_inputs(B, T, H, dk, dv, "bf16", s0_std=0.05, zg_mean=-1.0, seed=31), "bf16", "tcgen05")


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_prefill_head64_is_the_zero_padded_head128_problem(dk, dv):
    """The tensor-core kernel computes a head size of 64 as the 128-wide problem with zero channels
    (q = k = g = 0 past dk, v = 0 past dv).  Running that padded problem explicitly must give the
    same bits: the outputs' first dv columns, the state's top-left dk x dv block, and zeros elsewhere."""
    B, T, H = 2, 333, 3
    q, k, v, g, beta, S0 = gpu_inputs(B, T, H, dk, dv, "bf16", s0_std=0.05, zg_mean=-1.0, seed=32)
    o, ST = run_prefill((q, k, v, g, beta, S0), "tcgen05")

    def pad(x, d):
        out = torch.zeros(x.shape[:-1] + (128,), dtype=x.dtype, device=DEV)
        out[..., :d] = x
        return out.contiguous()

    S0p = torch.zeros((B, H, 128, 128), dtype=torch.float32, device=DEV)
    S0p[:, :, :dk, :dv] = S0
    op, STp = run_prefill((pad(q, dk), pad(k, dk), pad(v, dv), pad(g, dk), beta, S0p), "tcgen05")
    assert torch.equal(o, op[..., :dv])
    assert torch.equal(ST, STp[:, :, :dk, :dv])
    assert not torch.any(op[..., dv:]) and not torch.any(STp[:, :, dk:]) and not torch.any(STp[:, :, :, dv:])
