"""The fp64 oracle against its pins (closed forms, exact rationals, fixtures, brute force)."""
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.default())
