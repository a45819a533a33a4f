"""The CPU oracle against its pins (closed forms, invariants, library
routines, brute force); see ``pins.py`` for what each one fixes."""
import pytest

from pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(orc, pin):
    pin(orc)
