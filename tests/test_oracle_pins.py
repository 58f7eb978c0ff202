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



@pytest.mark.parametrize("coeffs", [
    [(3.4445, -4.7750, 2.0315)] * 5,
    [(1.5, -0.5, 0.0)] * 4,
    [(2.0, -9.0, 1.0), (3.4445, -4.7750, 2.0315)],
])
def test_emulation_structure_is_exact_without_rounding(coeffs):
    """The emulation path (stored A, a I + B, intermediate X) is the
    Newton-Schulz step itself once its rounding is the identity; the exact
    path is pinned by the closed forms above."""
    import numpy as np
    rng = np.random.default_rng(5)
    X = rng.standard_normal((24, 40))
    X /= np.linalg.norm(X)
    exact = mo.newton_schulz(X, coeffs)
    emu = mo.newton_schulz(X, coeffs, round_fn=lambda v: v)
    assert np.max(np.abs(emu - exact)) <= 1e-12 * max(1.0, np.max(np.abs(exact)))


def test_bf16_emulation_stays_near_exact():
    """With bf16 rounding at the stored points, five quintic steps stay
    within the working tolerance of the exact result (rounding 2^-9 per
    store, amplified by the polynomial's slope)."""
    import numpy as np
    rng = np.random.default_rng(11)
    X = rng.standard_normal((64, 96))
    X /= np.linalg.norm(X)
    coeffs = [(3.4445, -4.7750, 2.0315)] * 5
    exact = mo.newton_schulz(X, coeffs)
    emu = mo.newton_schulz(X, coeffs, round_fn=mo.bf16_round)
    assert np.max(np.abs(emu - exact)) < 2e-2
