"""The oracle checked against what the pages and mathematics fix (CPU only)."""
import pytest

import oracle.qwen3_ref as R
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("name", sorted(ALL_PINS))
def test_pin(name):
    ALL_PINS[name](R)
