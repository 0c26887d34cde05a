"""The CPU oracle against its pins (exact arithmetic, brute force, closed forms,
textbook special cases, invariants).  No GPU needed."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.default())
