"""The oracle passes every pin (CPU only)."""
import pytest

from oracle_pins import PINS


@pytest.mark.parametrize("name", sorted(PINS))
def test_oracle_pin(name):
    assert PINS[name](0), f"oracle fails pin {name}"
