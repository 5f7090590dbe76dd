"""The oracle against the pages' printed numbers, closed forms, invariants,
library routines and brute force (CPU only)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()
