"""Pin strength: each planted mistake in the oracle must break at least one pin.

The mistakes are planted in the oracle itself (CPU only) through its test hook;
see the "planted mistake N" markers in oracle/hils_oracle.c.
"""
import pytest

import pins
from oracle import oracle as orc

PLANTED = {
    1: "retrieval score without the 1/sqrt(d) scale",
    2: "query's own token masked out of its own chunk",
    3: "score ties resolved to the higher chunk index",
    4: "own chunk dropped from the fusion",
    6: "own chunk also ranked among the past candidates",
    7: "keys used in place of values",
    9: "one softmax over all selected tokens instead of per-chunk softmax + fusion",
    11: "each chunk scored with its neighbour's landmark",
}


@pytest.mark.parametrize("m", sorted(PLANTED), ids=lambda m: "mistake%d" % m)
def test_planted_mistake_is_caught(m):
    try:
        orc.set_mutant(m)
        res = pins.run_all()
    finally:
        orc.set_mutant(0)
    broken = [name for name, f in res.items() if f]
    assert broken, "planted mistake %d (%s) broke no pin" % (m, PLANTED[m])


def test_hook_off_again():
    orc.set_mutant(0)
    assert all(not f for f in pins.run_all().values())
