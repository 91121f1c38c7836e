"""The fp64 oracle against brute force, invariants, closed forms and the
hand-worked example (CPU only)."""
import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(orc, pin):
    assert orc.mutant == 0
    pin(orc)
