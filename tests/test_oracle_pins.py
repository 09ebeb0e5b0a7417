"""The fp64 oracle against closed forms, dense library solves, exact identities and
finite differences (see tests/oracle_checks.py for what pins what)."""
import pytest

import oracle
import oracle_checks as OC


@pytest.fixture(scope="module")
def ora():
    return oracle.get()


@pytest.mark.parametrize("check", OC.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(ora, check):
    check(ora)
