"""Backward pass on the GPU (hils_backward) against the float64 backward oracle (oracle/backward.py).

Gradients of sum(O * dO) through a fixed selection ("Hierarchical Sparse Attention Done Right", Sec. 3
Methodology, "Hierarchical softmax": the retrieval scores are trained through the fusion weights; a
chunk that is not selected gets no gradient).  The selection is the oracle's own (its forward pass on
the same inputs); the GPU receives it as its input, so both sides differentiate the same function.

Bound: the kernel computes in float32 from the exactly widened inputs (bf16 or float32), so every
gradient element is compared with max-abs error 1e-4 relative to the largest magnitude of its tensor
(at least 1): float32 rounding of sums over at most a few thousand contributions stays far below it,
for float32 and bf16 inputs alike.  K, V and L rows that no query reaches must be exactly zero.
"""
import numpy as np
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
import parity
from oracle import backward as bw
from oracle import oracle as orc
from synth import workloads as W
from synth.philox import f64_to_f32, f32_to_bf16_bits, bf16_bits_to_f64
from synth.workloads import Workload

pytestmark = pytest.mark.gpu

TOL = 1e-4


def wl(name, **kw):
    base = dict(B=1, H=4, Hkv=2, N=256, T=256, d=128, C=64, k=3, q_offset=0, dtype="bf16", seed=300,
                l_mode="chunkmean")
    base.update(kw)
    return Workload(name, **base)


CASES = [
    wl("f32_d64_c32_g2", N=300, T=300, d=64, C=32, k=3, dtype="f32", seed=301, input_scale=True, l_mode="iid"),
    wl("bf16_d128_c64_g4", B=2, H=8, Hkv=2, N=512, T=512, k=4, seed=302),
    wl("f32_chunked_offset", N=128, T=1024, q_offset=896, k=5, dtype="f32", seed=303),
    wl("bf16_decode", B=3, H=8, Hkv=2, N=1, T=3000, q_offset=2999, k=8, seed=304),
    wl("f32_k0_own_chunk_only", N=200, T=200, k=0, dtype="f32", seed=305),
    wl("bf16_k_more_than_visible", N=200, T=200, C=32, k=16, seed=306),
    wl("bf16_g16_c128", H=16, Hkv=1, N=400, T=400, C=128, k=2, seed=307),
]


def _dO(w):
    r = np.random.default_rng(w.seed + 11)
    x32 = f64_to_f32(r.standard_normal((w.B, w.H, w.N, w.d)))
    if w.dtype == "f32":
        return x32.astype(np.float64), x32
    bits = f32_to_bf16_bits(x32)
    return bf16_bits_to_f64(bits), bits


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_the_oracle(w):
    inp = W.full_inputs(w)
    arr = {k: v[0] for k, v in inp.items()}
    dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
    dO64, dOraw = _dO(w)
    dOd = parity.to_device(dOraw, w.dtype)
    fwd = orc.forward(arr["Q"], arr["K"], arr["V"], arr["L"], w.C, w.k, q_offset=w.q_offset)
    sel = fwd["sel"]
    sel_d = torch.from_numpy(np.ascontiguousarray(sel[..., :w.k]).astype(np.int32)).cuda() if w.k else None
    p = parity.problem_of(w)
    dQ = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.float32, device="cuda")
    dK = torch.full((w.B, w.Hkv, w.T, w.d), float("nan"), dtype=torch.float32, device="cuda")
    dV = torch.full_like(dK, float("nan"))
    dL = torch.full((w.B, w.Hkv, w.nL, w.d), float("nan"), dtype=torch.float32, device="cuda")
    hils.hils_backward(p, dev["Q"], dev["K"], dev["V"], dev["L"], sel_d, dOd, dQ, dK, dV, dL)
    assert hils.hils_sync_status() == hils.HILS_OK
    ref = bw.backward(arr["Q"], arr["K"], arr["V"], arr["L"], dO64, w.C, w.k, q_offset=w.q_offset, sel=sel)
    got = [t.double().cpu().numpy() for t in (dQ, dK, dV, dL)]
    for name, g, r in zip(("dQ", "dK", "dV", "dL"), got, ref):
        assert np.all(np.isfinite(g)), name
        bound = TOL * max(1.0, float(np.max(np.abs(r))))
        err = float(np.max(np.abs(g - r)))
        print(w.name, name, "max err %.3g (bound %.3g, max |ref| %.3g)" % (err, bound, float(np.max(np.abs(r)))))
        assert err <= bound, (name, err, bound)
    # rows of chunks no query reached: exactly zero
    for b in range(w.B):
        for g in range(w.Hkv):
            reached = set(int(c) for c in sel[b, g].ravel() if c >= 0)
            for c in range(w.nL):
                if c in reached:
                    continue
                assert not np.any(got[3][b, g, c]), ("dL", b, g, c)
                rows = slice(c * w.C, min((c + 1) * w.C, w.T))
                assert not np.any(got[1][b, g, rows]) and not np.any(got[2][b, g, rows]), ("dK/dV", b, g, c)
