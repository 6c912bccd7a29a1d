"""The oracle against closed forms, library special cases, hand-derived fixtures
and brute force (no GPU)."""
import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
