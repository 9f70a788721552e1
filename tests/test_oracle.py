"""Pins of the fp64 oracle (CPU only): closed forms, the lecture's invariants,
finite differences, a library special case and golden fixtures."""
import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(orc, pin):
    pin(orc)
