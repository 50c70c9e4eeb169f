"""The oracle checked against the absorption identity, rotary geometry, brute force,
library attention, the mask, the ring closed form and the cache-size closed forms."""

import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
