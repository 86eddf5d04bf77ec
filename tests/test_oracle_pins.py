"""The f64 oracle against brute force, closed forms and invariants (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(oracle_handle, pin):
    pin(oracle_handle)
