"""The CPU oracle against its pins (no GPU)."""
import pytest

from oracle import sla_oracle
from tests.oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(sla_oracle)
