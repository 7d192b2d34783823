"""The CPU oracle against its pins (facts fixed by the pages and by mathematics)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_round_bf16_matches_float32_conversion_and_ties():
    """The output rounding model: equals torch's bf16 conversion on float32 inputs,
    rounds exact ties to even, and rounds directly from float64 (no double rounding)."""
    import numpy as np
    import torch
    rng = np.random.default_rng(0)
    x32 = (rng.standard_normal(50000) * 7).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(oracle.round_bf16(x32.astype(np.float64)), ref)
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 1 + 2 ** -8 + 2 ** -40, 0.0, 3.0])
    want = np.array([1.0, 1 + 2 ** -6, -1.0, 1 + 2 ** -7, 0.0, 3.0])
    assert np.array_equal(oracle.round_bf16(x), want)


def test_half_ulp_bound_of_the_parity_check():
    """The rounding term of the parity bar: half a bf16 ulp at the binade of y (exact
    powers of two for y = 1, 1.5, 2, 0.75, -3), and every correctly rounded bf16 value
    lies within it of the exact value, with equality only at ties."""
    import numpy as np
    from helpers import half_ulp_bf16
    y = np.array([1.0, 1.5, 2.0, 0.75, -3.0, 0.0])
    assert np.array_equal(half_ulp_bf16(y), [2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -9, 2.0 ** -7, 0.0])
    rng = np.random.default_rng(5)
    x = rng.standard_normal(100000) * np.exp2(rng.integers(-20, 20, 100000))
    assert np.all(np.abs(oracle.round_bf16(x) - x) <= half_ulp_bf16(x))
    # a tie sits exactly half an ulp away
    t = np.array([1 + 2 ** -8])
    assert np.abs(oracle.round_bf16(t) - t)[0] == half_ulp_bf16(t)[0]
