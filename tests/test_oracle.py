"""The CPU oracle against its pins (hand-worked fixture, closed forms, exact
integer re-derivation, library special cases, brute force, invariants)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
