"""The float64 oracle against the facts that pin it (CPU only)."""
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS,
                         ids=[p.__name__ for p in oracle_pins.ALL_PINS])
def test_pin(pin):
    pin(oracle)
