"""The fp64 oracle against its pins (closed forms, invariants, library and brute-force special cases)."""
import pytest

import oracle.paged_attention as P
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(P)


def test_bytes_per_token():
    pins.pin_bytes_per_token()
