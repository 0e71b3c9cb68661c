"""The oracle against its pins (CPU only).  See tests/pins.py for what pins what."""
import pytest

from pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)
