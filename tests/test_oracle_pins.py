"""The fp64 oracle against hand-worked examples, closed forms, library routines
and the structural invariants of the MISA equations (CPU only)."""

import pytest

import oracle.misa_oracle as orc
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(orc)
