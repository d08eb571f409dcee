"""The CPU oracle against the pages' worked example, closed forms, invariants
and a contiguous numpy brute force (no GPU)."""
import pytest

from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()
