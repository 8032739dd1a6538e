"""The fp64 oracle against closed forms, invariants, golden values and finite differences."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=[p.__name__ for p in pins.ALL_PINS])
def test_oracle_pin(pin):
    compared = pin(oracle.default())
    assert compared > 0  # every pin must actually compare something
