"""The CPU oracle against its pins (closed forms, brute force, library routines)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)


def test_golden_files_parse():
    assert len(oracle_pins.read_lse_cases()) >= 20
    assert len(oracle_pins.read_combine_cases()) >= 7
