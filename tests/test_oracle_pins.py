"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import pins
from oracle import oracle as orc


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    orc.set_mutant(0)
    assert pin() == []


def test_tie_alternatives():
    shat = np.array([5.0, 1.0, 3.0, 3.0004, 2.0, 2.9995])
    # k=2: primary {0, 3}; band around 3.0004 with eps 1e-3 holds 2, 3, 5 -> three choices for one slot
    alts = orc.tie_alternatives(shat, 6, 2, 1e-3)
    assert [a.tolist() for a in alts] == [[0, 3], [0, 2], [0, 5]]  # primary first, then the others in index order
    assert len(orc.tie_alternatives(shat, 6, 2, 1e-5)) == 1
    assert orc.tie_alternatives(np.zeros(40), 40, 10, 1e-3, max_alts=8) is None
    assert [a.tolist() for a in orc.tie_alternatives(shat, 1, 3, 1e-3)] == [[0, -1, -1]]
