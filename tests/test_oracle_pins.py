"""The fp64 oracle against hand derivations, brute force and textbook reductions (CPU)."""
import pytest

from oracle import moe_oracle
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(moe_oracle)
