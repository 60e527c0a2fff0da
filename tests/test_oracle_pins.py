"""The fp64 oracle against the pins listed in tests/oracle_checks.py (CPU only)."""
import pytest

import oracle_checks as C


@pytest.mark.parametrize("check", C.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check()
