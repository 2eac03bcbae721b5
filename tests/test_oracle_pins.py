"""The fp64 oracle against its pins (CPU only)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS + [pins.pin_golden_regression],
                         ids=lambda f: f.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)
