"""The fp64 oracle against its pins (brute force, closed forms, invariants); CPU only."""
import pytest

from tests import pins


@pytest.mark.parametrize("name", list(pins.PINS))
def test_pin(oracle, name):
    assert pins.PINS[name](oracle), f"oracle fails pin {name}"
