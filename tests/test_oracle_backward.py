"""Pins of the backward-pass oracle (oracle/backward.py) against facts that do not come from it.

  * central finite differences of sum(O * dO) through the forward oracle, with the selection unchanged
    by the perturbation (checked), for elements of Q, K, V and L;
  * the dense reduction: chunk size 1, landmarks = keys and k covering every chunk make the forward pass
    dense causal attention, so the gradients of Q and V equal torch's autograd of its float64
    scaled_dot_product_attention, the gradient of L equals that of K there, and K itself gets none
    (a one-token chunk's softmax is constant);
  * one chunk (N = T = C): causal attention with a single fusion slot, so L gets no gradient and
    Q, K, V get causal attention's;
  * constant values: the output does not depend on Q, K or L, so their gradients vanish;
  * unselected chunks: K, V and L rows of chunks no query selected get no gradient.
Planted mistakes in the oracle (a softmax backward without its mean term, in either softmax; no path
through the fusion weights; a dropped scale; a missing fusion weight) must each break a pin.
"""
import math

import numpy as np
import pytest
import torch

from oracle import backward as bw
from oracle import oracle as orc


def _problem(seed, B, H, Hkv, T, d, C, l_equals_k=False):
    r = np.random.default_rng(seed)
    Q = r.standard_normal((B, H, T, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    L = K.copy() if l_equals_k else r.standard_normal((B, Hkv, -(-T // C), d))
    dO = r.standard_normal((B, H, T, d))
    return Q, K, V, L, dO


def _sdpa_grads(Q, K, V, dO, scale):
    G = Q.shape[1] // K.shape[1]
    q = torch.from_numpy(Q).requires_grad_()
    k = torch.from_numpy(K).requires_grad_()
    v = torch.from_numpy(V).requires_grad_()
    o = torch.nn.functional.scaled_dot_product_attention(q, k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1),
                                                         is_causal=True, scale=scale)
    (o * torch.from_numpy(dO)).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


def pin_finite_differences():
    fails = []
    B, H, Hkv, T, d, C, k = 1, 4, 2, 40, 6, 8, 2
    Q, K, V, L, dO = _problem(3, B, H, Hkv, T, d, C)
    scale = 1.0 / math.sqrt(d)
    base = orc.forward(Q, K, V, L, C, k, scale=scale, nthreads=1)
    dQ, dK, dV, dL = bw.backward(Q, K, V, L, dO, C, k, scale=scale, sel=base["sel"])
    grads = {"Q": dQ, "K": dK, "V": dV, "L": dL}
    r = np.random.default_rng(4)
    eps = 1e-6
    checked = 0
    for name in ("Q", "K", "V", "L"):
        arrs = {"Q": Q, "K": K, "V": V, "L": L}
        X = arrs[name]
        for _ in range(12):
            idx = tuple(int(r.integers(0, n)) for n in X.shape)
            vals = []
            for sgn in (1, -1):
                Xp = X.copy()
                Xp[idx] += sgn * eps
                a = dict(arrs, **{name: Xp})
                res = orc.forward(a["Q"], a["K"], a["V"], a["L"], C, k, scale=scale, nthreads=1)
                if not np.array_equal(res["sel"], base["sel"]):
                    break
                vals.append(float((res["O"] * dO).sum()))
            if len(vals) < 2:
                continue          # the perturbation moved the selection: not a smooth point
            fd = (vals[0] - vals[1]) / (2 * eps)
            checked += 1
            if not abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)):
                fails.append("finite difference d%s%s: oracle %.9g vs %.9g" % (name, idx, grads[name][idx], fd))
    if checked < 40:
        fails.append("finite differences: only %d of 48 points were smooth" % checked)
    return fails


def pin_dense_reduction():
    fails = []
    B, H, Hkv, T, d = 1, 4, 2, 24, 8
    Q, K, V, L, dO = _problem(5, B, H, Hkv, T, d, 1, l_equals_k=True)
    scale = 1.0 / math.sqrt(d)
    dQ, dK, dV, dL = bw.backward(Q, K, V, L, dO, 1, T, scale=scale)
    gQ, gK, gV = _sdpa_grads(Q, K, V, dO, scale)
    for name, got, want in (("Q", dQ, gQ), ("V", dV, gV), ("L", dL, gK), ("K", dK, np.zeros_like(gK))):
        e = float(np.abs(got - want).max())
        if not e <= 1e-11:
            fails.append("dense reduction d%s: max err %.3g" % (name, e))
    return fails


def pin_one_chunk():
    fails = []
    C = 16
    Q, K, V, L, dO = _problem(7, 1, 2, 1, C, 8, C)
    scale = 1.0 / math.sqrt(8)
    dQ, dK, dV, dL = bw.backward(Q, K, V, L, dO, C, 3, scale=scale)
    gQ, gK, gV = _sdpa_grads(Q, K, V, dO, scale)
    for name, got, want in (("Q", dQ, gQ), ("K", dK, gK), ("V", dV, gV), ("L", dL, np.zeros_like(dL))):
        e = float(np.abs(got - want).max())
        if not e <= 1e-11:
            fails.append("one chunk d%s: max err %.3g" % (name, e))
    return fails


def pin_constant_values():
    fails = []
    B, H, Hkv, T, d, C, k = 1, 4, 2, 50, 8, 8, 2
    Q, K, V, L, dO = _problem(9, B, H, Hkv, T, d, C)
    V = np.broadcast_to(np.random.default_rng(10).standard_normal(d), V.shape).copy()
    dQ, dK, dV, dL = bw.backward(Q, K, V, L, dO, C, k)
    for name, gr in (("Q", dQ), ("K", dK), ("L", dL)):
        if not float(np.abs(gr).max()) <= 1e-12:
            fails.append("constant values: d%s not zero (%.3g)" % (name, float(np.abs(gr).max())))
    return fails


def pin_unselected_chunks():
    fails = []
    B, H, Hkv, T, d, C, k = 1, 2, 1, 64, 8, 8, 1
    Q, K, V, L, dO = _problem(11, B, H, Hkv, T, d, C)
    Q = Q[:, :, 40:]
    dO = dO[:, :, 40:]
    res = orc.forward(Q, K, V, L, C, k, q_offset=40, nthreads=1)
    used = set(int(c) for c in res["sel"].ravel() if c >= 0)
    dQ, dK, dV, dL = bw.backward(Q, K, V, L, dO, C, k, q_offset=40, sel=res["sel"])
    for c in range(-(-T // C)):
        if c in used:
            continue
        rows = slice(c * C, (c + 1) * C)
        if np.abs(dK[0, 0, rows]).max() or np.abs(dV[0, 0, rows]).max() or np.abs(dL[0, 0, c]).max():
            fails.append("unselected chunk %d has a gradient" % c)
    if len(used) == -(-T // C):
        fails.append("every chunk selected: the pin checks nothing")
    return fails


PINS = [pin_finite_differences, pin_dense_reduction, pin_one_chunk, pin_constant_values, pin_unselected_chunks]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_backward_pin_holds(pin):
    assert pin() == []


PLANTED = {
    21: "fusion-weight softmax backward without its weighted mean",
    22: "no gradient through the fusion weights",
    23: "chunk softmax backward without its weighted mean",
    24: "scale dropped from the key gradient",
    25: "fusion weight missing from the value gradient",
}


@pytest.mark.parametrize("m", sorted(PLANTED), ids=lambda m: "mistake%d" % m)
def test_planted_mistake_in_the_backward_is_caught(m):
    broken = []
    try:
        bw.set_mutant(m)
        for pin in PINS:
            if pin():
                broken.append(pin.__name__)
    finally:
        bw.set_mutant(0)
    assert broken, "planted mistake %d (%s) broke no pin" % (m, PLANTED[m])
