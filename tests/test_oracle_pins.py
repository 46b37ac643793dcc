"""The float64 oracle against facts outside itself (see tests/pins.py)."""
import pytest

from pins import ALL_CHECKS


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check()
