"""The oracle against its pins (brute force, closed forms, invariants,
textbook values, the pages' printed numbers)."""
import pytest

from oracle import moe as orc
from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(orc)
