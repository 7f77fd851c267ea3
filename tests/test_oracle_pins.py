"""The fp64 oracle checked against closed forms, hand-worked examples, library
routes, finite differences and invariants (CPU only)."""
import pytest

import oracle
from tests import _pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", _pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
