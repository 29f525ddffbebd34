"""The float64 oracle against its pins (CPU only)."""
import pytest

import oracle.attention as oracle_mod
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle_mod)
