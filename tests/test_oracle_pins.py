"""The CPU oracle against closed forms, a library routine, the pages' invariants and
worked examples, and an independent numpy statement (no GPU needed)."""
import pytest

from tests import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)
