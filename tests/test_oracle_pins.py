"""The fp64 oracle against hand-solved examples, brute force, closed forms,
a textbook MoE and invariants (see oracle_pins.py)."""
import pytest

from oracle import moe_zc_ref
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(moe_zc_ref)
