"""The oracle against the pins (printed numbers, closed forms, invariants,
library routines for the special cases that reduce to them)."""
import pytest

from oracle import ds4a_oracle as O
from pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(O)
