"""The float64 oracle against its pins (CPU only)."""
import pytest

import oracle
from oracle_pins import ALL_PINS, COMPOSITION_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.lib())


@pytest.mark.parametrize("pin", COMPOSITION_PINS, ids=lambda p: p.__name__)
def test_oracle_composition_pin(pin):
    pin(oracle)
