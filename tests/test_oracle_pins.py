"""The CPU oracle against independent facts (see tests/pins.py)."""
import pytest

import pins


@pytest.mark.parametrize("check", pins.ALL, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check()
