"""The oracle against its pins (CPU only)."""
import pytest

import oracle_pins as P
from oracle import fpx_oracle as O


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(O)
