"""The CPU oracle against its pins (hand-worked format example, closed forms,
brute force, invariants). Runs without a GPU."""
import pytest

import pins_lib


@pytest.mark.parametrize("check", pins_lib.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(orc, check):
    check()
