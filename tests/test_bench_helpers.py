"""bench.py's byte counts and recorded ncu traffic (CPU).

The roofline divides algorithmic bytes per launch by the launch time, so the counts are pinned here
to figures derived by hand: per token-head, prefill reads q, k, g (dk each), v (dv) and beta and
writes o (dv), all bf16: 2 * (3 * 128 + 128) + 2 + 2 * 128 = 1282 B at d = 128; per head it reads S0
and writes S_T, 64 KiB each.  A decode head-step reads and writes the 64 KiB fp32 state and moves
1026 B of token inputs and 256 B of output.
"""
import bench


def test_prefill_bytes_of_the_k3_workload():
    assert bench.prefill_alg_bytes(4, 8192, 96, 128, 128) == 4 * 8192 * 96 * 1282 + 2 * 4 * 96 * 65536
    assert bench.prefill_alg_bytes(4, 8192, 96, 128, 128) == 4_083_154_944
    # the long-context workload starts from a zero state: S_T is written, S0 is not read
    assert bench.prefill_alg_bytes(1, 65536, 96, 128, 128, with_s0=False) == 65536 * 96 * 1282 + 96 * 65536


def test_decode_bytes_of_a_step():
    per_head_step = 2 * 65536 + 1026 + 256
    assert per_head_step == 132_354
    assert bench.decode_alg_bytes(256, 96, 128, 128) == 256 * 96 * per_head_step


def test_recorded_traffic_is_parsed_and_close_to_the_algorithmic_bytes():
    # a record counts only while the kernel sources it was captured on are unchanged
    for tag, alg in (("prefill_tc", bench.prefill_alg_bytes(4, 8192, 96, 128, 128)),
                     ("decode", bench.decode_alg_bytes(256, 96, 128, 128))):
        t = bench.recorded_traffic(tag)
        if t is not None:
            assert 0.95 * alg <= t <= 1.05 * alg, (tag, t, alg)


def test_kernel_source_hash_is_stable_and_short():
    a, b = bench.kernel_source_sha("prefill_tc"), bench.kernel_source_sha("prefill_tc")
    assert a == b and len(a) == 16 and a != bench.kernel_source_sha("decode")


def test_input_fingerprint_identifies_the_seeded_bytes():
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs, fingerprint
    a = make_prefill_inputs(1, 130, 2, 64, 64, "bf16", seed=3, s0_std=0.05)
    b = make_prefill_inputs(1, 130, 2, 64, 64, "bf16", seed=3, s0_std=0.05)
    c = make_prefill_inputs(1, 130, 2, 64, 64, "bf16", seed=4, s0_std=0.05)
    assert fingerprint(*a) == fingerprint(*b) and fingerprint(*a) != fingerprint(*c)
    # the same values in another dtype are other bytes
    assert fingerprint(a[0]) != fingerprint(a[0].float())


def test_batching_leg_shapes_and_bytes(monkeypatch):
    """The continuous-batching leg at tiny sizes on the CPU, with the library and CUDA events stubbed:
    the packed layout, the slot table and the byte counts it reports."""
    import types
    import torch

    class Event:
        def __init__(self, enable_timing=True):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 2.0

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    seen = {}

    def varlen(q, k, v, g, beta, cu, S0, o=None, S_T=None, stream=None):
        seen["varlen"] = (q.shape, v.shape, beta.shape, cu.dtype, int(cu[-1]), S0.shape, o.shape, S_T.shape)

    def paged(q, k, v, g, beta, pool, slots, stream=None):
        seen["paged"] = (q.shape, pool.shape, slots.dtype, len(set(slots.tolist())), int(slots.max()))

    kda = types.SimpleNamespace(kda_forward_varlen=varlen, kda_decode_step_paged=paged,
                                kda_get_device_status=lambda: 0)
    out = bench.measure_batching(kda, torch.device("cpu"), None, 0, types.SimpleNamespace(steps=3),
                                 H=2, d=64, nseq=5, max_len=100, batch=6, n_slots=16)
    tokens = out["packed_prefill"]["tokens"]
    assert seen["varlen"] == ((tokens, 2, 64), (tokens, 2, 64), (tokens, 2), torch.int32, tokens, (5, 2, 64, 64),
                              (tokens, 2, 64), (5, 2, 64, 64))
    # 642 B per token-head at d = 64 (q, k, g, v in and o out in bf16, and beta), 2 x 16 KiB of state per head
    assert out["packed_prefill"]["roofline"]["alg_bytes_per_launch"] == tokens * 2 * 642 + 5 * 2 * 2 * 64 * 64 * 4
    assert out["packed_prefill"]["roofline"]["alg_bytes_per_launch"] == bench.prefill_alg_bytes(1, tokens, 2, 64, 64) + \
        (5 - 1) * 2 * 2 * 64 * 64 * 4
    assert seen["paged"][:3] == ((6, 2, 64), (16, 2, 64, 64), torch.int32)
    assert seen["paged"][3] == 6 and seen["paged"][4] < 16            # distinct slots inside the pool
    assert out["paged_decode"]["roofline"]["alg_bytes_per_launch"] == bench.decode_alg_bytes(6, 2, 64, 64)


def test_long_split_leg_stacks_the_three_segment_runs(monkeypatch):
    """The long-context split leg at tiny sizes on the CPU with the library stubbed: one stacked launch of
    (first half from 0, second half from 0, second half with v = 0 and S0 = I), then the correction of
    the second half's outputs with the first half's final state, and the state composition."""
    import types
    import torch
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs

    class Event:
        def __init__(self, enable_timing=True):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 1.0

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    B, T, H, d = 1, 128, 2, 64
    lq = make_prefill_inputs(B, T, H, d, d, "bf16", seed=1)
    lo = torch.zeros((B, T, H, d), dtype=torch.bfloat16)
    lst = torch.ones((B, H, d, d))
    seen = {}

    def forward(q, k, v, g, beta, S0, o=None, S_T=None, stream=None):
        h = T // 2
        assert q.shape == (3 * B, h, H, d) and o.shape == (3 * B, h, H, d) and S_T.shape == (3 * B, H, d, d)
        assert torch.equal(q[0], lq[0][0, :h]) and torch.equal(q[1], lq[0][0, h:]) and torch.equal(q[2], lq[0][0, h:])
        assert torch.equal(v[1], lq[2][0, h:]) and not torch.any(v[2])
        assert not torch.any(S0[:2]) and torch.equal(S0[2], torch.eye(d).expand(H, d, d))
        o.zero_()
        S_T.copy_(lst.expand(3 * B, H, d, d))
        seen["forward"] = seen.get("forward", 0) + 1

    def correct(C, S_in, o_in, out=None, stream=None):
        seen["correct"] = (C.shape, S_in.shape, out.data_ptr() == o_in.data_ptr())

    def compose(M, S, N, out=None, stream=None):
        out.copy_(lst)
        seen["compose"] = (M.shape, S.shape, N.shape)

    kda = types.SimpleNamespace(kda_forward_chunked=forward, kda_output_correct=correct, kda_state_compose=compose,
                                kda_get_device_status=lambda: 0)
    LC = dict(B=B, T=T, H=H, dk=d, dv=d)
    out = bench.measure_long_split(kda, LC, lq, lo, lst, None, 3, 1.0)
    assert seen["correct"] == ((B, T // 2, H, d), (B, H, d, d), True)
    assert seen["compose"] == ((B, H, d, d), (B, H, d, d), (B, H, d, d))
    assert out["ctas"] == 3 * B * H and out["segments"] == 2 and out["max_rel_diff_state_vs_single_pass"] == 0.0
