"""The oracle against its pins (CPU only).  See tests/oracle_pins.py for what
each pin fixes and the passage it follows."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_chunked_form_is_itself_exact_against_brute_force():
    """The test-side chunked restatement is checked against the test-side brute
    force too, so a mistake shared by the oracle and one restatement shows."""
    import numpy as np
    x = P.rand_inputs([37], H=1, dk=5, dv=4, seed=91, s0_std=0.5)
    o_b, st = P.brute_force_chain(x["q"][:, 0], x["k"][:, 0], x["v"][:, 0], x["g"][:, 0],
                                  x["beta"][:, 0], x["s0"][0, 0])
    for C in (1, 8, 16, 37):
        o_c, s_c = P.chunked_chain(x["q"][:, 0], x["k"][:, 0], x["v"][:, 0], x["g"][:, 0],
                                   x["beta"][:, 0], x["s0"][0, 0], C)
        np.testing.assert_allclose(o_c, o_b, rtol=0, atol=1e-11)
        np.testing.assert_allclose(s_c, st[-1], rtol=0, atol=1e-11)
