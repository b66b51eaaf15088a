"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(oracle, pin):
    pin(oracle)


def test_numpy_half_rounding_is_direct():
    """The tests round the oracle's doubles to fp16 with numpy; that rounding
    must go straight from double (no double rounding through float32)."""
    v = np.float64(1.0 + 2.0**-11 + 2.0**-40)   # just above the fp16 tie
    assert float(v.astype(np.float16)) == 1.0 + 2.0**-10
    t = np.float64(1.0 + 2.0**-11)              # exact tie -> even
    assert float(t.astype(np.float16)) == 1.0
    t3 = np.float64(1.0 + 3 * 2.0**-11)         # tie between odd and even mantissa
    assert float(t3.astype(np.float16)) == 1.0 + 2 * 2.0**-10


def test_golden_parses():
    cases = P.parse_golden()
    assert {c["name"] for c in cases} == {"two_rows", "one_group_zero_point",
                                          "ffn_one_row", "lm_head_tie"}
