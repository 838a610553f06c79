"""Input generator checks (CPU): Philox known answers, rounding, random access, recipes."""
import os

import numpy as np

from synth import philox as P
from synth import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip() and l[0] != "#"]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = P.philox4x32_10(tuple(v[0:4]), tuple(v[4:6]))
        assert [int(x) for x in out] == v[6:10]


def test_bf16_rounding_closed_forms():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -2.5, 3.0e-39], dtype=np.float32)
    bits = P.f32_to_bf16_bits(x)
    back = P.bf16_bits_to_f64(bits)
    # ties to even, above-tie rounds up, exact values stay, subnormal keeps its top bits
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 4 * 2 ** -8
    assert back[3] == 1.0 + 2 ** -7 and back[4] == -2.5
    assert bits[5] == (np.array([3.0e-39], np.float32).view(np.uint32)[0] + 0x8000) >> 16


def test_random_access_matches_range():
    idx = np.array([0, 1, 2, 3, 1001, 77777, 2 ** 33 + 5], dtype=np.uint64)
    a = P.gaussian_at(7, 3, idx)
    r = P.gaussian_range(7, 3, 0, 4)
    assert np.array_equal(a[:4], r)
    b = P.gaussian_range(7, 3, 77770, 10)
    assert a[5] == b[7]
    z = P.gaussian_range(1, 1, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_workload_recipes():
    w = W.WORKLOADS["prefill_256k_needles"]
    for g in range(w.Hkv):
        nc = W.needle_chunks(w, g)
        assert len(nc) == 64 and len(set(nc.tolist())) == 64 and nc.min() >= 0 and nc.max() < w.T // w.C
        u = W.needle_u(w, g)
        assert abs(np.dot(u, u) - 1) < 1e-12
    # chunk-mean landmarks: mean of the rounded keys plus 0.1-scaled noise
    w2 = W.WORKLOADS["prefill_8k"]
    L, Lraw = W.l_rows(w2, 1, 3, 5, 7)
    K, _ = W.k_rows(w2, 1, 3, 5 * 64, 7 * 64)
    noise = (L - K.reshape(2, 64, -1).mean(axis=1)) / 0.1
    assert np.abs(noise).max() < 6 and 0.5 < noise.std() < 1.5
    assert Lraw.dtype == np.uint16
    # query needles
    q, _ = W.q_rows(w, 0, [0, 5], np.array([511, 512, 1024]))
    q0, _ = W.q_rows(w.with_(n_needles=0), 0, [0, 5], np.array([511, 512, 1024]))
    dq = q - q0
    assert np.abs(dq[:, 0]).max() == 0 and np.abs(dq[:, 1]).max() > 0.1
    # tiny fp32 workload is scaled by d^-1/4
    w1 = W.WORKLOADS["tiny_f32"]
    qq, raw = W.q_rows(w1, 0, [0], np.arange(1024))
    assert raw.dtype == np.float32 and abs(qq.std() - 64 ** -0.25) < 0.01
