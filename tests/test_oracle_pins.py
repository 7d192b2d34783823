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
