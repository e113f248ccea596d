"""The CPU oracle against brute force, a library routine, closed forms and
invariants (no GPU)."""

import pytest

import oracle
from tests.oracle_pins import PINS


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(lib, pin):
    pin(lib)
