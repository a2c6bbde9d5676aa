"""The CPU oracle against its pins (closed forms, library routines,
brute force, hand-worked values).  CPU only."""
import pytest

import oracle.kq_oracle as o
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(o)
