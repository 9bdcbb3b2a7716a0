"""Every mistake planted in the oracle (built with -DORC_MUTANT=n) must trip at
least one pin, so the pins would notice such a mistake in the oracle itself."""
import inspect
import math

import numpy as np
import pytest

from oracle import oracle as oracle_mod
from oracle.oracle import Oracle
import oracle_pins

MUTANTS = {
    1: "correction weight n_j dropped",
    2: "threshold as a linear fraction of the max",
    3: "query head mapped to KV group h % Hkv",
    4: "strict comparison at the threshold",
    5: "block mean divided by the block size, not the row count",
    6: "causal mask excludes the diagonal token",
    7: "score without the softmax scale",
    8: "diagonal block not forced",
    9: "mean key used as the correction value",
    10: "value scale ignored",
    11: "LSE without the row max",
    12: "chunk: causal mask relative to the chunk start, not the position",
    13: "chunk: partial first q-block mean divided by rows before the chunk too",
    14: "chunk: pruned blocks of the cached prefix get no correction",
    15: "variance variant: the full logit variance added instead of half of it",
    16: "isotropic variance variant: variances summed, not averaged, over the dimensions",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=[MUTANTS[m] for m in sorted(MUTANTS)])
def test_mutant_is_caught(mutant):
    orc = Oracle(mutant)
    assert orc.lib.orc_mutant_id() == mutant
    tripped = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            tripped.append(pin.__name__)
    assert tripped, f"planted mistake '{MUTANTS[mutant]}' passes every pin"


# Planted mistakes in the mask comparison's band (oracle.oracle.near_threshold),
# each one textual edit of the function's source.
NEAR_MUTANTS = {
    "band without the absolute floor of one": (
        "band = rel * np.maximum(1.0, np.abs(thr))", "band = rel * np.abs(thr)"),
    "band scaled by ln(alpha) instead of the threshold": (
        "band = rel * np.maximum(1.0, np.abs(thr))", "band = rel * np.maximum(1.0, np.abs(0.0 * thr + math.log(alpha)))"),
    "union over the wrong head axis (group h % Hkv)": (
        "reshape(nblk, kept_shape_groups, G, nb_max).any(axis=2)",
        "reshape(nblk, G, kept_shape_groups, nb_max).any(axis=1)"),
    "distance to the row max instead of the threshold": (
        "np.abs(s - thr[:, :, None])", "np.abs(s - m[:, :, None])"),
}


@pytest.mark.parametrize("name", sorted(NEAR_MUTANTS))
def test_near_threshold_mutant_is_caught(name):
    old, new = NEAR_MUTANTS[name]
    src = inspect.getsource(oracle_mod.near_threshold)
    assert old in src, f"mutation site '{old}' not found in near_threshold"
    ns = {"np": np, "math": math}
    exec(src.replace(old, new), ns)
    with pytest.raises(AssertionError):
        oracle_pins.pin_near_threshold(ns["near_threshold"])
