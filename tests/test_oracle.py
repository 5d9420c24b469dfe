"""The fp64 oracle against its pins (hand-worked fixtures, library special cases,
invariants). CPU only."""
import pytest

from oracle import bsa_oracle as O
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(O)
