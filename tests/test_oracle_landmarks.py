"""Pins of the oracle's landmark generation (landmark = the chunk's keys weighted by the landmark
query's softmax over them; bias = the entropy of that softmax).

The facts come from outside the oracle: closed forms for uniform and one-hot weights, the variational
identity of log-sum-exp (for any distribution p over the keys, sum_t p_t s_t + H(p) <= log sum_t
exp(s_t), with equality exactly at p = softmax(s)), and invariances."""
import math

import numpy as np
import pytest

from oracle import oracle as orc


def _keys(seed, B, Hkv, T, d):
    return np.random.default_rng(seed).standard_normal((B, Hkv, T, d))


def test_uniform_query_gives_the_mean_key_and_log_c():
    B, Hkv, T, d, C = 2, 2, 50, 8, 16          # a partial last chunk of 2 keys
    K = _keys(1, B, Hkv, T, d)
    nL = -(-T // C)
    L, beta = orc.landmarks(K, np.zeros((B, Hkv, nL, d)), C)
    for c in range(nL):
        rows = min(C, T - c * C)
        assert np.max(np.abs(L[:, :, c] - K[:, :, c * C:c * C + rows].mean(axis=2))) <= 1e-14
        assert np.max(np.abs(beta[:, :, c] - math.log(rows))) <= 1e-14


def test_one_dominant_key_gives_that_key_and_zero_entropy():
    B, Hkv, T, d, C = 1, 1, 32, 8, 8
    K = _keys(2, B, Hkv, T, d)
    nL = T // C
    U = np.zeros((B, Hkv, nL, d))
    for c in range(nL):
        U[0, 0, c] = 4000.0 * K[0, 0, c * C + 3]   # key 3 of every chunk dominates by far
    L, beta = orc.landmarks(K, U, C)
    for c in range(nL):
        assert np.max(np.abs(L[0, 0, c] - K[0, 0, c * C + 3])) <= 1e-9
        assert beta[0, 0, c] <= 1e-9


def test_surrogate_is_a_lower_bound_of_the_chunk_mass_tight_at_the_landmark_query():
    B, Hkv, T, d, C = 1, 2, 64, 16, 16
    r = np.random.default_rng(3)
    K = r.standard_normal((B, Hkv, T, d))
    nL = T // C
    U = r.standard_normal((B, Hkv, nL, d))
    scale = 1.0 / math.sqrt(d)
    L, beta = orc.landmarks(K, U, C, scale=scale)
    for g in range(Hkv):
        for c in range(nL):
            keys = K[0, g, c * C:(c + 1) * C]
            for q in [U[0, g, c]] + list(r.standard_normal((6, d))):
                s = scale * keys @ q
                lse = float(np.max(s) + np.log(np.sum(np.exp(s - np.max(s)))))
                surrogate = scale * float(q @ L[0, g, c]) + float(beta[0, g, c])
                assert surrogate <= lse + 1e-12
            s = scale * keys @ U[0, g, c]
            lse = float(np.max(s) + np.log(np.sum(np.exp(s - np.max(s)))))
            assert abs(scale * float(U[0, g, c] @ L[0, g, c]) + float(beta[0, g, c]) - lse) <= 1e-12


def test_order_of_keys_inside_a_chunk_does_not_matter():
    B, Hkv, T, d, C = 1, 1, 48, 8, 16
    r = np.random.default_rng(4)
    K = r.standard_normal((B, Hkv, T, d))
    U = r.standard_normal((B, Hkv, T // C, d))
    L1, b1 = orc.landmarks(K, U, C)
    K2 = K.copy()
    for c in range(T // C):
        K2[0, 0, c * C:(c + 1) * C] = K[0, 0, c * C + r.permutation(C)]
    L2, b2 = orc.landmarks(K2, U, C)
    assert np.max(np.abs(L1 - L2)) <= 1e-13 and np.max(np.abs(b1 - b2)) <= 1e-13


@pytest.mark.parametrize("C", [1, 7])
def test_entropy_stays_between_zero_and_log_c(C):
    B, Hkv, T, d = 2, 1, 70, 4
    r = np.random.default_rng(5 + C)
    K = r.standard_normal((B, Hkv, T, d)) * 3.0
    U = r.standard_normal((B, Hkv, -(-T // C), d)) * 3.0
    _, beta = orc.landmarks(K, U, C)
    assert np.all(beta >= -1e-15) and np.all(beta <= math.log(C) + 1e-12)


PINS = [test_uniform_query_gives_the_mean_key_and_log_c, test_one_dominant_key_gives_that_key_and_zero_entropy,
        test_surrogate_is_a_lower_bound_of_the_chunk_mass_tight_at_the_landmark_query,
        test_order_of_keys_inside_a_chunk_does_not_matter]

PLANTED = {
    15: "scale dropped from the landmark query's scores",
    16: "entropy with the wrong sign",
    17: "bias log C whatever the scores",
}


@pytest.mark.parametrize("m", sorted(PLANTED), ids=lambda m: "mistake%d" % m)
def test_planted_mistake_in_the_landmarks_is_caught(m):
    broken = []
    try:
        orc.set_mutant(m)
        for pin in PINS + [lambda: test_entropy_stays_between_zero_and_log_c(7)]:
            try:
                pin()
            except AssertionError:
                broken.append(getattr(pin, "__name__", "entropy bounds"))
    finally:
        orc.set_mutant(0)
    assert broken, "planted mistake %d (%s) broke no pin" % (m, PLANTED[m])
