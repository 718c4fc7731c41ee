"""The CPU oracle against what fixes it from outside: hand-worked fixtures, closed forms,
library routines, invariants and pure-Python brute force (see ``oracle_pins.py``)."""
import pytest

import oracle.oracle as O
import oracle_pins as P


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(O)
