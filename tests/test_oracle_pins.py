"""The float64 oracle against facts that mathematics and library routines fix (CPU only)."""
import pytest

import oracle_pins
from oracle import oracle as O


@pytest.fixture(scope="module")
def lib():
    return O.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)
