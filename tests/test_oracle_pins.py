"""The oracle against hand-derived values, closed forms, invariants and
independent numpy brute force (no GPU)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
