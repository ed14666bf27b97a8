"""The CPU oracle against its pins (closed forms, worked fixtures, brute force,
invariants and library routines); see tests/pins.py."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
