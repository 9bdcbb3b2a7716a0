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


def test_float_build_agrees_with_the_double_build():
    """The float build only times the CPU baseline; it is the same code as the parity
    build, so on a small layer it keeps the same kept lists and its outputs stay within
    float rounding of the double build's."""
    import numpy as np
    from workloads import make_workload
    wl = make_workload([700, 300], 8, 2, alpha=0.1, seed=5)
    a = Oracle().run(wl, want_scores=True)
    b = Oracle(fp32=True).run(wl, want_scores=True)
    assert b["o"].dtype == np.float32 and a["o"].dtype == np.float64
    assert (a["kept_cnt"] == b["kept_cnt"]).all() and (a["kept_idx"] == b["kept_idx"]).all()
    assert np.abs(a["o"] - b["o"]).max() < 1e-4
    assert np.abs(a["lse"] - b["lse"]).max() < 1e-4
