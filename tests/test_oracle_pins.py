"""The CPU oracle against its pins (closed forms, hand-derived examples,
dense and library statements of the same attention, invariants, finite
differences).  No GPU."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)
