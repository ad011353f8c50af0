"""The tensor-core prefill and the decode kernel on the five measured workloads (GPU).

Small cases compare every element with the oracle; at full size the comparison runs on
sampled heads the oracle can afford (whole sequences for those heads), as configured for
the benchmark launch.  Tolerance: max |x - ref| / max |ref| <= 2e-2 (bf16), 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200.inputs import (PREFILL_CONFIGS, DECODE_CONFIG, make_config_inputs,
                                                             make_prefill_inputs, make_decode_inputs)
from helpers import max_rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def head_slice(x, b, h):
    return x[b:b + 1, :, h:h + 1].contiguous()


def oracle_heads(inputs, heads):
    """Oracle on the selected (b, h) heads, stacked along the head axis so they run in parallel."""
    q, k, v, g, beta, S0 = inputs
    idx_b = [b for b, _ in heads]
    idx_h = [h for _, h in heads]
    pick = lambda x: torch.stack([x[b, :, h] for b, h in zip(idx_b, idx_h)], dim=1)[None].contiguous()
    s0 = None if S0 is None else torch.stack([S0[b, h] for b, h in zip(idx_b, idx_h)])[None].contiguous()
    o_ref, ST_ref = oracle.forward(pick(q), pick(k), pick(v), pick(g), pick(beta), s0, nthreads=0)
    return [(o_ref[:, :, j:j + 1], ST_ref[:, j:j + 1]) for j in range(len(heads))]


@pytest.mark.parametrize("T", [64, 128, 191, 320, 1000])
@pytest.mark.parametrize("regime", ["recipe", "worst_decay", "no_decay", "adversarial"])
def test_tc_matches_oracle(T, regime):
    q, k, v, g, beta, S0 = make_prefill_inputs(2, T, 3, 128, 128, "bf16", seed=T, s0_std=0.1, device=DEV)
    if regime == "worst_decay":
        g = torch.full_like(g, -5.0)
    elif regime == "no_decay":
        g = (g * 0.01).contiguous()      # long memory: the state carries across many chunks
    elif regime == "adversarial":
        # g = -5 on tokens 33..48 of every chunk, ~0 elsewhere: column factors of the block-1 x
        # block-0 rectangle underflow while nearby pair factors stay of order one
        g = torch.full_like(g, -1e-3)
        for c0 in range(0, T, 64):
            g[:, c0 + 33:c0 + 49] = -5.0
    o, ST = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl="tcgen05")
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0, nthreads=0)
    assert max_rel_err(to_np(o), o_ref) <= 2e-2
    assert max_rel_err(to_np(ST), ST_ref) <= 2e-2


def test_tc_agrees_with_fp32_simt_kernel():
    q, k, v, g, beta, S0 = make_prefill_inputs(1, 700, 4, 128, 128, "bf16", seed=3, s0_std=0.05, device=DEV)
    o1, S1 = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl="tcgen05")
    o2, S2 = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl="simt")
    torch.cuda.synchronize()
    assert max_rel_err(to_np(o1), to_np(o2)) <= 2e-2
    assert max_rel_err(to_np(S1), to_np(S2)) <= 2e-2


def test_config_h32_t4k_full():
    """B1 T4096 H32 d128 bf16, S0 = 0: every output element against the oracle."""
    cfg = PREFILL_CONFIGS["h32_t4k"]
    inputs = make_config_inputs(cfg, device=DEV)
    o, ST = kda.kda_forward_chunked(*inputs)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref = oracle.forward(*inputs, nthreads=0)
    assert max_rel_err(to_np(o), o_ref) <= 2e-2
    assert max_rel_err(to_np(ST), ST_ref) <= 2e-2


def test_config_small_fp32_full():
    cfg = PREFILL_CONFIGS["small_fp32"]
    inputs = make_config_inputs(cfg, device=DEV)
    o, ST = kda.kda_forward_chunked(*inputs)
    torch.cuda.synchronize()
    o_ref, ST_ref = oracle.forward(*inputs)
    assert max_rel_err(to_np(o), o_ref) <= 1e-4
    assert max_rel_err(to_np(ST), ST_ref) <= 1e-4


def test_config_k3_b4_t8k_sampled_heads():
    """The benchmark's K3 workload (B4 T8192 H96), launched whole; 8 heads checked end to end."""
    cfg = PREFILL_CONFIGS["k3_b4_t8k"]
    inputs = make_config_inputs(cfg, device=DEV)
    o, ST = kda.kda_forward_chunked(*inputs)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    heads = [(0, 0), (0, 95), (1, 17), (1, 48), (2, 63), (2, 5), (3, 94), (3, 31)]
    for (b, h), (o_ref, ST_ref) in zip(heads, oracle_heads(inputs, heads)):
        assert max_rel_err(to_np(head_slice(o, b, h)), o_ref) <= 2e-2, (b, h)
        assert max_rel_err(to_np(ST[b:b + 1, h:h + 1]), ST_ref) <= 2e-2, (b, h)


def test_config_k3_t64k_prefix_and_final_state():
    """B1 T65536 H96: o on the first 4096 tokens and the full-length S_T, for sampled heads."""
    cfg = PREFILL_CONFIGS["k3_t64k"]
    inputs = make_config_inputs(cfg, device=DEV)
    o, ST = kda.kda_forward_chunked(*inputs)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    heads = [(0, 0), (0, 41), (0, 77), (0, 95)]
    for (b, h), (o_ref, ST_ref) in zip(heads, oracle_heads(inputs, heads)):
        assert max_rel_err(to_np(head_slice(o, b, h)[:, :4096]), o_ref[:, :4096]) <= 2e-2, (b, h)
        assert max_rel_err(to_np(head_slice(o, b, h)), o_ref) <= 2e-2, (b, h)
        assert max_rel_err(to_np(ST[b:b + 1, h:h + 1]), ST_ref) <= 2e-2, (b, h)


def test_config_decode_full_batch():
    """256 sequences x 96 heads, 128x128 fp32 states, updated in place: 3 steps, every element."""
    D = DECODE_CONFIG
    gen = torch.Generator(device=DEV)
    gen.manual_seed(D.seed)
    S = torch.zeros((D.batch, D.H, D.dk, D.dv), dtype=torch.float32, device=DEV)
    S_ref = np.zeros((D.batch, D.H, D.dk, D.dv))
    for _ in range(3):
        x = make_decode_inputs(D.batch, D.H, D.dk, D.dv, D.dtype, gen=gen, device=DEV)
        o = kda.kda_decode_step(*x, S)
        o_ref = oracle.decode_step(*x, S_ref, nthreads=0)
        torch.cuda.synchronize()
        assert max_rel_err(to_np(o), o_ref) <= 2e-2
    assert max_rel_err(to_np(S), S_ref) <= 2e-2
