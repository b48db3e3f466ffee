"""The CPU oracle against its pins (closed forms, library routines, brute force,
invariants); see oracle_pins.py for what each pin checks and why."""
import pytest

import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(0)
