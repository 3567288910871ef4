"""The CPU oracle against its pins (see tests/pins.py for what each pin rests on)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=[p.__name__ for p in pins.ALL_PINS])
def test_pin(orc, pin):
    pin(orc)
