"""The oracle's gate forward/backward against closed forms, finite differences,
an independent autograd restatement and invariants (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.GATE_PINS, ids=lambda f: f.__name__)
def test_gate_pin(oracle_lib, pin):
    pin(oracle_lib)
