"""The fp64 oracle against the pages' worked examples, closed forms, SDPA and brute force."""
import pytest

import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS + pins.SLOW_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check, oracle_module):
    check(oracle_module)
