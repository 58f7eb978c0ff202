"""The fp64 oracle against its pins (closed forms, invariants, SVD, exact
rational arithmetic).  CPU only."""
import pytest

import oracle.muon_oracle as mo
import oracle.polar_express as pe
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(mo)


def test_polar_express_table():
    pins.pin_polar_express_table(pe)


def test_bf16_round_matches_definition():
    """bf16 rounding helper of the emulation mode: nearest representable
    value with ties to even, checked on hand-built bit patterns."""
    import numpy as np
    one = 1.0
    ulp = 2.0 ** -7                    # bf16 spacing in [1, 2)
    xs = np.array([one, one + ulp / 2, one + ulp / 2 + 2 ** -20,
                   one + 3 * ulp / 2, -(one + ulp / 4)])
    want = np.array([one, one, one + ulp, one + 2 * ulp, -one])
    assert np.array_equal(mo.bf16_round(xs), want)
