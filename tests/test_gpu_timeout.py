"""Failure detection without a GPU fault: a device-side wait is made to run out on purpose.

The tensor-core prefill bounds every mbarrier wait in wall time.  The test hook
kda_debug_set_wait_fault(1, t) makes the operand warps skip their first hand-off to the
recurrence warps, so a wait is certain to expire after t; the kernel must then report
KDA_ERR_TIMEOUT through the device status word, finish (drain its tensor-core and TMA work,
free tensor memory) instead of hanging, and leave the CUDA context usable.  Nothing traps,
faults or spins forever.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_forward_b200 as kda
from linear_attention_recurrence_forward_b200 import STATUS
from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
from helpers import max_rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [50, 200])
def test_timed_out_wait_is_reported_and_context_survives(T):
    inputs = make_prefill_inputs(1, T, 2, 128, 128, "bf16", seed=1, s0_std=0.05, device="cuda")
    assert kda.kda_get_device_status() == 0
    kda.kda_debug_set_wait_fault(1, 20_000_000)  # every wait limited to 20 ms
    try:
        t0 = time.perf_counter()
        kda.kda_forward_chunked(*inputs, impl="tcgen05")
        status = kda.kda_get_device_status()
        elapsed = time.perf_counter() - t0
    finally:
        kda.kda_debug_set_wait_fault(0)
    assert status == STATUS["KDA_ERR_TIMEOUT"]
    assert elapsed < 5.0
    # the status word was cleared by the read, and the context still computes correctly
    o, ST = kda.kda_forward_chunked(*inputs, impl="tcgen05")
    assert kda.kda_get_device_status() == 0
    o_ref, ST_ref = oracle.forward(*inputs)
    assert max_rel_err(o.double().cpu().numpy(), o_ref) <= 2e-2
    assert max_rel_err(ST.double().cpu().numpy(), ST_ref) <= 2e-2
