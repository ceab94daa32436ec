"""The fp64 oracle against facts that do not come from it (CPU only)."""
import pytest

import oracle.rs_oracle as rs_oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(rs_oracle)
