"""The fp64 oracle against hand-worked values, closed forms, invariants and an
independent library computation (see oracle_pins.py for each pin's source)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
