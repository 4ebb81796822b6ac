"""The oracle against its pins (CPU only).  See tests/oracle_pins.py."""
import pytest

from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(oracle_lib, check):
    check(oracle_lib)
