"""The CPU oracle against printed values, closed forms, invariants, library
routines and brute force (no GPU)."""
import pytest

import oracle.tpa_oracle as O
from tests.oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin(O)
