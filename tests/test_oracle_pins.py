"""The float64 oracle against closed forms, library routines, the LTI
convolutional mode, chunk-split invariance and brute-force bracketing."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)
