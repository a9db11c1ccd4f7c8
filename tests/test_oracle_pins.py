"""The CPU oracle against its pins (hand-worked examples, closed forms, brute
force and textbook attention on special cases).  CPU only."""

import pytest

from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
