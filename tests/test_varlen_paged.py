"""Packed variable-length prefill and paged-state decode (continuous batching).

Every packed sequence must give what it gives alone (the oracle on that sequence), the o rows
outside every range stay untouched, equal lengths give bitwise what the [B, T, H, d] layout
gives, and invalid device-side offsets or slots are reported through the status word without
touching memory they do not own.  Paged decode must equal the oracle on the gathered states,
leave inactive slots alone, and equal the plain decode bitwise for an identity slot table.
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS
from helpers import max_rel_err

OK, INVALID, UNSUPPORTED, MISALIGNED = (STATUS[n] for n in
                                        ("KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                         "KDA_ERR_MISALIGNED"))
TOL = {"bf16": 2e-2, "fp32": 1e-4}

# ---------------------------------------------------------------------- C ABI checks (CPU)

BASE = 0x7F0000000000
SZ = 1 << 30


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrence_forward_b200 import build
    build.build()
    return kda.lib()


def varlen(L, p, N=4, T=1000, H=2, dk=128, dv=128, dtype=0, impl=0):
    q, k, v, g, beta, cu, S0, o, ST = p
    return L.kda_forward_varlen(q, k, v, g, beta, cu, S0, o, ST, N, T, H, dk, dv, dtype, impl, None)


def ptrs():
    return [BASE + i * SZ for i in range(9)]


def test_varlen_rejects_bad_arguments(L):
    assert varlen(L, ptrs(), N=0) == INVALID
    p = ptrs(); p[5] = None
    assert varlen(L, p) == INVALID                       # cu_seqlens is required
    p = ptrs(); p[5] += 4
    assert varlen(L, p) == MISALIGNED
    assert varlen(L, ptrs(), dk=96) == UNSUPPORTED
    assert varlen(L, ptrs(), impl=9) == INVALID
    assert varlen(L, ptrs(), T=-1) == INVALID
    p = ptrs(); p[7] = p[0] + 4096                       # o inside q
    assert varlen(L, p) == INVALID
    p = ptrs(); p[5] = p[7] + 64                         # cu_seqlens inside o
    assert varlen(L, p) == INVALID
    p = ptrs(); p[8] = p[6] + 4096                       # S_T partly over S0
    assert varlen(L, p) == INVALID
    assert varlen(L, ptrs(), dtype=1, impl=1) == UNSUPPORTED   # the tensor-core kernel is bf16 only


def paged(L, p, B=4, n_slots=8, H=2, dk=128, dv=128, dtype=0):
    q, k, v, g, beta, S, slots, o = p[:8]
    return L.kda_decode_step_paged(q, k, v, g, beta, S, n_slots, slots, o, B, H, dk, dv, dtype, None)


def test_paged_decode_rejects_bad_arguments(L):
    p = ptrs(); p[6] = None
    assert paged(L, p) == INVALID                        # slots are required
    assert paged(L, ptrs(), n_slots=0) == INVALID
    p = ptrs(); p[6] += 4
    assert paged(L, p) == MISALIGNED
    p = ptrs(); p[6] = p[5] + 1024                       # slot table inside the pool
    assert paged(L, p) == INVALID
    assert paged(L, ptrs(), dk=80) == UNSUPPORTED


# ---------------------------------------------------------------------- GPU

gpu = pytest.mark.gpu


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def packed_case(lengths, H, d, dtype, seed=0, lead=0, tail=0):
    """Packed inputs for sequences of the given lengths (plus `lead` / `tail` unused tokens)."""
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    T_total = lead + sum(lengths) + tail
    q, k, v, g, beta, _ = make_prefill_inputs(1, T_total, H, d, d, dtype, seed=seed, device="cuda")
    q, k, v, g, beta = (x[0].contiguous() for x in (q, k, v, g, beta))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]) + lead, dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed + 1)
    S0 = (torch.randn((len(lengths), H, d, d), generator=gen, device="cuda") * 0.05).contiguous()
    return q, k, v, g, beta, cu, S0


@gpu
@pytest.mark.parametrize("dtype,impl,d", [("bf16", "tcgen05", 128), ("bf16", "tcgen05", 64), ("bf16", "simt", 128),
                                          ("fp32", "simt", 64)])
def test_packed_sequences_match_the_oracle_one_by_one(dtype, impl, d):
    lengths = [1, 63, 64, 65, 200, 0, 130, 7]
    q, k, v, g, beta, cu, S0 = packed_case(lengths, 3, d, dtype, seed=2)
    o, ST = kda.kda_forward_varlen(q, k, v, g, beta, cu, S0, impl=impl)
    torch.cuda.synchronize()
    assert kda.kda_get_device_status() == 0
    bounds = cu.cpu().numpy()
    for n, T in enumerate(lengths):
        s0, s1 = bounds[n], bounds[n + 1]
        sl = [x[s0:s1][None] for x in (q, k, v, g, beta)]
        o_ref, ST_ref = oracle.forward(*sl, S0[n:n + 1])
        assert max_rel_err(np64(o[s0:s1]), o_ref[0]) <= TOL[dtype], n
        assert max_rel_err(np64(ST[n]), ST_ref[0]) <= TOL[dtype], n


@gpu
@pytest.mark.parametrize("impl", ["tcgen05", "simt"])
def test_equal_lengths_match_the_batched_layout_bitwise(impl):
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    B, T, H = 3, 200, 2
    q, k, v, g, beta, S0 = make_prefill_inputs(B, T, H, 128, 128, "bf16", seed=4, s0_std=0.05, device="cuda")
    o_b, ST_b = kda.kda_forward_chunked(q, k, v, g, beta, S0, impl=impl)
    flat = [x.reshape((B * T,) + tuple(x.shape[2:])).contiguous() for x in (q, k, v, g, beta)]
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device="cuda")
    o_p, ST_p = kda.kda_forward_varlen(*flat, cu, S0, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(o_p.reshape(B, T, H, 128), o_b) and torch.equal(ST_p, ST_b)


@gpu
@pytest.mark.parametrize("impl", ["tcgen05", "simt"])
def test_rows_outside_the_ranges_are_untouched(impl):
    lengths = [70, 5, 129]
    q, k, v, g, beta, cu, S0 = packed_case(lengths, 2, 128, "bf16", seed=6, lead=5, tail=7)
    o = torch.full((q.shape[0], 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    kda.kda_forward_varlen(q, k, v, g, beta, cu, S0, o=o, impl=impl)
    torch.cuda.synchronize()
    assert bool((o[:5] == 7.0).all()) and bool((o[-7:] == 7.0).all())
    assert not bool((o[5:-7] == 7.0).all())


@gpu
@pytest.mark.parametrize("impl", ["tcgen05", "simt"])
@pytest.mark.parametrize("fault", ["past_end", "overlap", "negative"])
def test_invalid_offsets_are_reported_not_followed(impl, fault):
    """Offsets that are not one valid layout (a range past the tokens, two overlapping ranges, a
    negative start) are reported and no sequence is processed: every S_T is its S0 and no o row is
    written, so no two CTAs ever write the same rows."""
    lengths = [100, 60, 80]
    q, k, v, g, beta, cu, S0 = packed_case(lengths, 2, 128, "bf16", seed=8)
    bad = cu.clone()
    if fault == "past_end":
        bad[3] = q.shape[0] + 50    # sequence 2 runs past the tokens
    elif fault == "overlap":
        bad[1], bad[2] = 120, 90    # sequence 1 is [120, 90) (backwards); 0 = [0, 120) and 2 = [90, 240) overlap
    else:
        bad[0] = -4
    assert kda.kda_get_device_status() == 0
    o = torch.full((q.shape[0], 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    o, ST = kda.kda_forward_varlen(q, k, v, g, beta, bad, S0, o=o, impl=impl)
    assert kda.kda_get_device_status() == STATUS["KDA_ERR_INVALID_ARG"]
    assert torch.equal(ST, S0)                           # every sequence processed as empty
    assert bool((o == 7.0).all())                        # nothing written
    o, ST = kda.kda_forward_varlen(q, k, v, g, beta, cu, S0, impl=impl)
    assert kda.kda_get_device_status() == 0              # valid offsets: the word was cleared by the read
    for n in range(3):
        s0, s1 = int(cu[n]), int(cu[n + 1])
        o_ref, ST_ref = oracle.forward(*[x[s0:s1][None] for x in (q, k, v, g, beta)], S0[n:n + 1])
        assert max_rel_err(np64(o[s0:s1]), o_ref[0]) <= 2e-2
        assert max_rel_err(np64(ST[n]), ST_ref[0]) <= 2e-2


def decode_inputs(B, H, d, dtype, seed):
    from linear_attention_recurrence_forward_b200.inputs import make_decode_inputs
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    return make_decode_inputs(B, H, d, d, dtype, gen=gen, device="cuda")


@gpu
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64)])
def test_paged_decode_matches_the_oracle(dtype, d):
    B, H, n_slots = 6, 3, 10
    slots = torch.tensor([3, -1, 7, 0, 9, 5], dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1)
    pool = (torch.randn((n_slots, H, d, d), generator=gen, device="cuda") * 0.1).contiguous()
    pool_before = pool.clone()
    ref_pool = np64(pool).copy()
    o = torch.full((B, H, d), 3.0, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    for step in range(3):
        q, k, v, g, beta = decode_inputs(B, H, d, dtype, seed=10 + step)
        kda.kda_decode_step_paged(q, k, v, g, beta, pool, slots, o=o)
        torch.cuda.synchronize()
        act = [b for b in range(B) if int(slots[b]) >= 0]
        idx = [int(slots[b]) for b in act]
        S_ref = np.ascontiguousarray(ref_pool[idx])
        sel = [x[act] for x in (q, k, v, g, beta)]
        o_ref = oracle.decode_step(*sel, S_ref)
        ref_pool[idx] = S_ref
        assert max_rel_err(np64(o[act]), o_ref) <= TOL[dtype]
        assert bool((o[1] == 3.0).all())                 # the inactive sequence's output is untouched
    assert max_rel_err(np64(pool), ref_pool) <= TOL[dtype]
    untouched = [s for s in range(n_slots) if s not in (3, 7, 0, 9, 5)]
    assert torch.equal(pool[untouched], pool_before[untouched])
    assert kda.kda_get_device_status() == 0


@gpu
def test_paged_decode_with_identity_slots_equals_plain_decode():
    B, H, d = 5, 4, 128
    gen = torch.Generator(device="cuda")
    gen.manual_seed(2)
    S = (torch.randn((B, H, d, d), generator=gen, device="cuda") * 0.1).contiguous()
    S2 = S.clone()
    q, k, v, g, beta = decode_inputs(B, H, d, "bf16", seed=3)
    o1 = kda.kda_decode_step(q, k, v, g, beta, S)
    o2 = kda.kda_decode_step_paged(q, k, v, g, beta, S2, torch.arange(B, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S, S2)


@gpu
def test_paged_decode_reports_an_out_of_range_slot():
    B, H, d = 3, 2, 128
    pool = torch.zeros((4, H, d, d), device="cuda")
    q, k, v, g, beta = decode_inputs(B, H, d, "bf16", seed=5)
    slots = torch.tensor([0, 4, 2], dtype=torch.int32, device="cuda")   # 4 is past the pool
    kda.kda_decode_step_paged(q, k, v, g, beta, pool, slots)
    assert kda.kda_get_device_status() == STATUS["KDA_ERR_INVALID_ARG"]
    assert bool((pool[1] == 0).all()) and bool((pool[3] == 0).all())
