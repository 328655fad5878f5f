"""The CPU oracle against its pins (no GPU).

Each check is defined in ``tests/oracle_pins.py``; see there for what pins
what.  These run on the oracle built from ``oracle/oracle.c``."""
import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(orc, check):
    check(orc)
