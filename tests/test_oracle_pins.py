"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""
import pytest

from oracle import poet_oracle as O
from tests import oracle_pins


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    assert check(O)
