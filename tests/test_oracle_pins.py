"""The CPU oracle against its pins (hand-worked goldens, closed forms, special
cases and an independent numpy restatement)."""
import pytest

import oracle
from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.load())
