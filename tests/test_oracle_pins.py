"""The float64 oracle against the pages' figures, closed forms, library attention and
special cases (CPU only)."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.load())
