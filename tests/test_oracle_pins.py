"""The oracle pinned to the pages' worked numbers and to mathematics (CPU)."""
import pytest

from oracle_checks import ALL_CHECKS


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()
