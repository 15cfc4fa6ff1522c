"""The mixed bit-width key cache part of the CPU oracle against what the abstract and mathematics
fix (runs without a GPU)."""
import pytest

import gtq_pins as P


@pytest.mark.parametrize("pin", P.GTQ_PINS, ids=[f.__name__ for f in P.GTQ_PINS])
def test_gtq_pin(pin):
    pin()
