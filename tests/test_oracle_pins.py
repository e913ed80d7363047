"""The CPU oracle against its pins (brute force, library routines, closed
forms, invariants).  No GPU needed."""
import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=[p.__name__ for p in P.ALL_PINS])
def test_pin(pin):
    pin()
