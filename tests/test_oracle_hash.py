"""The oracle's n-gram hash and table-row gather against their pins (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.HASH_PINS, ids=lambda f: f.__name__)
def test_hash_pin(oracle_lib, pin):
    pin(oracle_lib)
