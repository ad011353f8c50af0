"""I12: the chunk algebra the prefill kernel is built on reproduces the token recurrence.

The fp64 chunk model (tests/chunk_model.py) must agree with the oracle to ~1e-12 for any
chunk and sub-block size, with ragged tails, a nonzero initial state and the worst-case
decay g = -5 on every channel (where unfactored exponents over a 64-token chunk would
overflow).  With bf16 operands emulated at the kernel's rounding points it must stay well
inside the 2e-2 bf16 tolerance.
"""
import numpy as np
import pytest

import oracle
from chunk_model import kernel_inverse, chunk_forward
from helpers import max_rel_err, random_problem


@pytest.mark.parametrize("C,sub", [(64, 32), (64, 16), (32, 16), (16, 16)])
@pytest.mark.parametrize("worst_decay", [False, True])
def test_chunk_form_matches_oracle(C, sub, worst_decay):
    rng = np.random.default_rng(7)
    q, k, v, g, beta, S0 = random_problem(rng, 1, 150, 2, 16, 12)
    if worst_decay:
        g = np.full_like(g, -5.0)
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0, nthreads=2)
    o, ST = chunk_forward(q, k, v, g, beta, S0, C=C, sub=sub)
    assert max_rel_err(o, o_ref) < 1e-11, max_rel_err(o, o_ref)
    assert max_rel_err(ST, ST_ref) < 1e-11, max_rel_err(ST, ST_ref)


def test_chunk_form_slow_decay_with_state():
    rng = np.random.default_rng(8)
    q, k, v, g, beta, S0 = random_problem(rng, 1, 200, 1, 32, 32)
    g = g * 0.02                                    # nearly no forgetting: the state carries far
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0, nthreads=2)
    o, ST = chunk_forward(q, k, v, g, beta, S0, C=64, sub=32)
    assert max_rel_err(o, o_ref) < 1e-11 and max_rel_err(ST, ST_ref) < 1e-11


@pytest.mark.parametrize("zg_mean", [0.0, -2.0, -6.0])
def test_bf16_operands_stay_inside_tolerance(zg_mean):
    rng = np.random.default_rng(9)
    q, k, v, g, beta, S0 = random_problem(rng, 1, 320, 1, 64, 64)
    g = -5.0 / (1.0 + np.exp(-(rng.standard_normal(g.shape) + zg_mean)))
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0, nthreads=2)
    o, ST = chunk_forward(q, k, v, g, beta, S0, C=64, sub=32, bf16=True, offdiag_ref="row_middle",
                          solve="kernel")
    # half the 2e-2 bf16 tolerance, before the final bf16 rounding of o
    assert max_rel_err(o, o_ref) < 1e-2, max_rel_err(o, o_ref)
    assert max_rel_err(ST, ST_ref) < 1e-2, max_rel_err(ST, ST_ref)


def adversarial_decay(T, dk, chunk=64):
    """g = -5 on tokens 33..48 of every chunk and ~0 elsewhere: the pattern that makes the
    block-1 x block-0 column factors e^{Gam_48 - Gam_j} underflow while nearby pair factors stay large."""
    g = np.full((1, T, 1, dk), -1e-3)
    for c0 in range(0, T, chunk):
        g[:, c0 + 33:c0 + 49] = -5.0
    return g


@pytest.mark.parametrize("pattern", ["recipe", "adversarial", "all_minus5"])
def test_kernel_factorisation_stays_close_to_oracle(pattern):
    """The kernel factors the block-1 x block-0 rectangle at token 48 and flushes column factors
    below the fp32 range.  In exact arithmetic otherwise, the dropped terms are each below
    e^{-7.3} of a unit product; the whole effect must stay under 1e-3 of max|o| and max|S|."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta, S0 = random_problem(rng, 1, 256, 1, 32, 32)
    if pattern == "adversarial":
        g = adversarial_decay(256, 32)
    elif pattern == "all_minus5":
        g = np.full_like(g, -5.0)
    o_ref, ST_ref = oracle.forward(q, k, v, g, beta, S0, nthreads=2)
    o, ST = chunk_forward(q, k, v, g, beta, S0, C=64, sub=32, offdiag_ref="row_middle")
    assert max_rel_err(o, o_ref) < 1e-3, max_rel_err(o, o_ref)
    assert max_rel_err(ST, ST_ref) < 1e-3, max_rel_err(ST, ST_ref)


def test_kernel_inverse_is_the_inverse_in_exact_arithmetic():
    """The doubling and block-distance recurrences give (I + A)^-1 exactly (no rounding)."""
    rng = np.random.default_rng(12)
    A = np.tril(rng.standard_normal((64, 64)) * 0.3, -1)
    X = kernel_inverse(A, lambda x: x)
    assert np.max(np.abs(X - np.linalg.inv(np.eye(64) + A))) < 1e-10
    # a plausible slip (one doubling round fewer) is caught
    N = A[:16, :16]
    short = (np.eye(16) - N) @ (np.eye(16) + N @ N) @ (np.eye(16) + np.linalg.matrix_power(N, 4))
    assert np.max(np.abs(short - np.linalg.inv(np.eye(16) + N))) > 1e-6
