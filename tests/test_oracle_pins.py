"""The CPU oracle against facts other than itself (see pins.py). CPU only."""

import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(o, pin):
    pin(o)
