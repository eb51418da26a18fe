"""The oracle against its pins (CPU only): a library attention routine, closed forms,
hand-derived golden values under tests/golden/ and invariants of the definitions."""

import pytest

from oracle import flux_oracle as orc
from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(orc)
