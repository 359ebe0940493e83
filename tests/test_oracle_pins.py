"""The fp64 oracle checked against hand-worked values, closed forms,
invariants and library routines (CPU only)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin()
