"""The CPU oracle against its pins (hand example, brute force, closed forms,
invariants); see tests/pins.py for what each pin fixes."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(None)
