"""The oracle against what the pages and mathematics fix (CPU only)."""
import numpy as np
import pytest

import oracle
from oracle_pins import ALL_PINS


def _fwd(q, k, v, g, beta, S0):
    return oracle.forward(q, k, v, g, beta, S0, nthreads=2)


def _dec(q, k, v, g, beta, S):
    return oracle.decode_step(q, k, v, g, beta, S, nthreads=2)


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(_fwd, _dec, np.random.default_rng(1234))


def test_oracle_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.forward(np.zeros((1, 2, 1, 0)), np.zeros((1, 2, 1, 0)), np.zeros((1, 2, 1, 3)),
                       np.zeros((1, 2, 1, 0)), np.zeros((1, 2, 1)))


def test_oracle_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(0)
    S0 = rng.standard_normal((2, 3, 4, 5))
    z = np.zeros((2, 0, 3, 4))
    o, ST = oracle.forward(z, z, np.zeros((2, 0, 3, 5)), z, np.zeros((2, 0, 3)), S0)
    assert o.shape == (2, 0, 3, 5)
    assert np.array_equal(ST, S0)


def test_oracle_threads_do_not_change_results():
    from helpers import random_problem
    q, k, v, g, beta, S0 = random_problem(np.random.default_rng(5), 2, 33, 5, 8, 8)
    o1, S1 = oracle.forward(q, k, v, g, beta, S0, nthreads=1)
    o4, S4 = oracle.forward(q, k, v, g, beta, S0, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)
