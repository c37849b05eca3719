"""The CPU oracle against its pins (library casts, brute force, closed forms,
exact results within the fp32 bound).  No GPU needed."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(oracle_mod, pin):
    pin(oracle_mod)
