"""The CPU oracle against the pages' worked numbers, closed forms, brute force,
special cases and an independent torch restatement (no GPU needed)."""
import pytest

from oracle import moe_oracle as O
from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(O)
