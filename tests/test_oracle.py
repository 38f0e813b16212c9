"""The oracle against its pins (CPU only).  See oracle_pins.py for what each
pin checks and why it is independent of the oracle's own code."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)
