"""The fp64 oracle against facts fixed outside it (pages, closed forms,
invariants, brute force, black-box CPU library routines)."""

import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle)
