"""Plausible mistakes planted in copies of the oracle (on the CPU) must each fail a pin.

This checks the pins, not the oracle: every mutant below is a one-line slip someone
could make when writing the recurrence (gate after the prediction, dropped beta, read-out
from the old state, wrong sign, transposed state access, inverted gate, a 1/sqrt(d)
query scale, an exclusive decay), and at least one pin must catch each.
"""
import numpy as np
import pytest

import oracle
from oracle_pins import ALL_PINS

DECAY = ("    for (i = 0; i < dk; ++i) {\n        double a = exp(g[i]);\n"
         "        for (c = 0; c < dv; ++c) S[i * dv + c] *= a;\n    }\n")

MUTANTS = {
    # apply the gate after the prediction instead of before it
    "decay_after_prediction": [(DECAY, ""),
                               ("    /* S <- S + k u^T */\n", DECAY + "    /* S <- S + k u^T */\n")],
    "beta_dropped": [("p[c] = beta * (v[c] - p[c]);", "p[c] = (v[c] - p[c]);")],
    "sign_flipped": [("p[c] = beta * (v[c] - p[c]);", "p[c] = beta * (v[c] + p[c]);")],
    "inverted_gate": [("double a = exp(g[i]);", "double a = exp(-g[i]);")],
    "query_scaled": [("o[c] += S[i * dv + c] * q[i];", "o[c] += S[i * dv + c] * q[i] / sqrt((double)dk);")],
    "transposed_prediction": [("p[c] += S[i * dv + c] * k[i];", "p[c] += S[c * dv + i] * k[i];")],
    # read out before the rank-1 update (o_t = S'^T q with the decayed old state)
    "readout_before_update": [
        ("    /* S <- S + k u^T */\n    for (i = 0; i < dk; ++i)\n        for (c = 0; c < dv; ++c) S[i * dv + c] += k[i] * p[c];\n"
         "    /* o = S^T q */\n    for (c = 0; c < dv; ++c) o[c] = 0.0;\n    for (i = 0; i < dk; ++i)\n"
         "        for (c = 0; c < dv; ++c) o[c] += S[i * dv + c] * q[i];\n",
         "    for (c = 0; c < dv; ++c) o[c] = 0.0;\n    for (i = 0; i < dk; ++i)\n"
         "        for (c = 0; c < dv; ++c) o[c] += S[i * dv + c] * q[i];\n"
         "    for (i = 0; i < dk; ++i)\n        for (c = 0; c < dv; ++c) S[i * dv + c] += k[i] * p[c];\n")],
    # control: a comment edit, nothing observable changes
    "control_comment_only": [("/* prediction p = S^T k */", "/* prediction */")],
}
# The last entry is a control that changes nothing observable; it must pass every pin.
CONTROL = "control_comment_only"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    src = oracle.source_text()
    for old, new in MUTANTS[name]:
        assert old in src, f"mutation anchor for {name} not found in the oracle source"
        src = src.replace(old, new, 1)
    lib = oracle.build_variant(src, str(tmp_path / f"lib_{name}.so"))

    def fwd(q, k, v, g, beta, S0):
        return oracle.forward(q, k, v, g, beta, S0, nthreads=1, lib=lib)

    def dec(q, k, v, g, beta, S):
        return oracle.decode_step(q, k, v, g, beta, S, nthreads=1, lib=lib)

    failed = []
    for pin in ALL_PINS:
        try:
            pin(fwd, dec, np.random.default_rng(1234))
        except AssertionError:
            failed.append(pin.__name__)
    if name == CONTROL:
        assert not failed, f"control mutant must pass all pins, failed {failed}"
    else:
        assert failed, f"no pin caught mutant {name}"
