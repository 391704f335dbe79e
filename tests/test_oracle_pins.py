"""The fp64 oracle against its pins (hand-worked examples, closed forms,
invariants, a hand-enumerated index table and torch's float64 SDPA)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.load())
