"""The CPU oracle against its pins (no GPU needed)."""
import pytest

from pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(oracle, pin):
    pin(oracle)
