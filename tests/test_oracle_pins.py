"""The CPU oracle against its pins (no GPU)."""
import pytest

from oracle.oracle import Oracle
import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return Oracle()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=[p.__name__ for p in oracle_pins.ALL_PINS])
def test_pin(orc, pin):
    pin(orc)


def test_near_threshold_band():
    from oracle.oracle import near_threshold
    oracle_pins.pin_near_threshold(near_threshold)
