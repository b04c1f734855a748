"""The oracle against its pins (CPU only)."""
import pytest

import oracle_pins
import ttq_oracle


@pytest.fixture(scope="module")
def O():
    return ttq_oracle.get()


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(O, check):
    check(O)
