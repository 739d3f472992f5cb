"""The CPU oracle against its pins (hand values, float64 library routines,
invariants, brute force).  CPU only."""
import pytest

from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)
