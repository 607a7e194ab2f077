"""The CPU oracle against closed forms, library routines, invariants and the pages' worked example."""
import pytest

import oracle
from oracle_pins import ALL_CHECKS


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__[len("check_"):])
def test_pin(lib, check):
    check(lib)
