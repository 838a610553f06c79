"""GPU vs oracle on prefill shapes whose selection bookkeeping leaves room for one value slot only.

The tensor-core prefill kernel streams values through two 32 KB slots when its shared memory allows
and through one otherwise (larger k and query tiles with more rows per query: G = 1 with
k = 21..31, G = 2 with k = 32..47, G = 4 with k = 43..63).  With one slot the value ring and the
P buffers must still be reused in order; these cases check every query group of such shapes,
including a ragged tail and an odd chunk union, against the oracle with the bounds of the other
parity suites.
"""
import pytest

import parity
from synth.workloads import Workload

pytestmark = pytest.mark.gpu


def wl(name, **kw):
    base = dict(B=1, H=4, Hkv=2, N=512, T=512, d=128, C=64, k=4, q_offset=0, dtype="bf16", seed=140,
                l_mode="chunkmean")
    base.update(kw)
    return Workload(name, **base)


CASES = [
    wl("g1_k24_one_value_slot", H=2, Hkv=2, N=64 * 40 + 21, T=64 * 40 + 21, k=24, seed=141),
    wl("g2_k40_one_value_slot", H=4, Hkv=2, N=64 * 50 + 3, T=64 * 50 + 3, k=40, seed=142, l_mode="iid"),
    wl("g4_k48_one_value_slot", H=8, Hkv=2, N=64 * 60 + 9, T=64 * 60 + 9, k=48, seed=143),
    wl("g4_k48_chunked_offset", H=8, Hkv=2, N=700, T=64 * 70, q_offset=64 * 70 - 700, k=48, seed=144),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_parity_one_value_slot(w):
    st, _ = parity.run_small(w)
    print(w.name, {k: v for k, v in st.items() if k != "fail"})
    assert st["fail"] == [], st["fail"][:5]
