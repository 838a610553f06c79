"""Pins of the oracle's extension for the next rows of the method: a chunk-aligned local window
(always attended, never a retrieval candidate) and a per-chunk bias of the retrieval score.

Each fact below comes from outside the oracle: the method without the extension (window of one
chunk, no bias), torch's scaled_dot_product_attention on dense and banded masks, brute-force
selection, and algebra (softmax shift invariance)."""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import oracle as orc


def _problem(seed, B, H, Hkv, T, d, C, l_equals_k=False):
    r = np.random.default_rng(seed)
    Q = r.standard_normal((B, H, T, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    L = K.copy() if l_equals_k else r.standard_normal((B, Hkv, -(-T // C), d))
    return Q, K, V, L


def _sdpa(Q, K, V, scale, mask):
    """mask [T, T] bool, True = attend."""
    G = Q.shape[1] // K.shape[1]
    q = torch.from_numpy(Q)
    k = torch.from_numpy(K).repeat_interleave(G, dim=1)
    v = torch.from_numpy(V).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask),
                                                            scale=scale).numpy()


def test_one_chunk_window_without_bias_is_the_method():
    Q, K, V, L = _problem(3, 2, 4, 2, 300, 16, 32)
    a = orc.forward(Q, K, V, L, C=32, k=3, nthreads=2)
    b = orc.forward_window(Q, K, V, L, C=32, k=3, wc=1, nthreads=2)
    assert np.array_equal(a["sel"], b["sel"])
    assert np.max(np.abs(a["O"] - b["O"])) <= 1e-15
    assert np.max(np.abs(a["w"] - b["w"])) <= 1e-15


def test_window_covering_every_chunk_is_dense_causal_attention():
    # chunk size 1 and landmarks = keys: a chunk is one token and its retrieval score is the token
    # logit, so fusing every visible chunk is causal softmax attention
    T, d = 37, 8
    Q, K, V, L = _problem(5, 1, 4, 2, T, d, 1, l_equals_k=True)
    scale = 1.0 / math.sqrt(d)
    res = orc.forward_window(Q, K, V, L, C=1, k=2, wc=T, scale=scale, nthreads=2)
    ref = _sdpa(Q, K, V, scale, np.tril(np.ones((T, T), dtype=bool)))
    assert np.max(np.abs(res["O"] - ref)) <= 1e-12


def test_window_only_is_sliding_window_attention():
    # chunk size 1, landmarks = keys, no retrieval: each query attends to its last W tokens
    T, d, W = 40, 8, 7
    Q, K, V, L = _problem(7, 2, 2, 1, T, d, 1, l_equals_k=True)
    scale = 1.0 / math.sqrt(d)
    res = orc.forward_window(Q, K, V, L, C=1, k=0, wc=W, scale=scale, nthreads=2)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    ref = _sdpa(Q, K, V, scale, (j <= i) & (j > i - W))
    assert np.max(np.abs(res["O"] - ref)) <= 1e-12


def test_window_plus_full_retrieval_is_dense():
    T, d = 30, 8
    Q, K, V, L = _problem(9, 1, 2, 2, T, d, 1, l_equals_k=True)
    scale = 1.0 / math.sqrt(d)
    res = orc.forward_window(Q, K, V, L, C=1, k=T, wc=4, scale=scale, nthreads=2)
    ref = _sdpa(Q, K, V, scale, np.tril(np.ones((T, T), dtype=bool)))
    assert np.max(np.abs(res["O"] - ref)) <= 1e-12


def test_window_and_retrieved_chunks_are_disjoint_and_ordered():
    C, k, wc, T = 8, 3, 3, 200
    Q, K, V, L = _problem(11, 1, 2, 1, T, 8, C)
    res = orc.forward_window(Q, K, V, L, C=C, k=k, wc=wc, nthreads=2)
    for i in range(T):
        ci = i // C
        sel = [int(c) for c in res["sel"][0, 0, i]]
        top, win = sel[:k], sel[k:]
        assert win == [c if c >= 0 else -1 for c in range(ci - wc + 1, ci + 1)]
        n_cand = max(ci - wc + 1, 0)
        real = [c for c in top if c >= 0]
        assert len(real) == min(k, n_cand) and all(0 <= c < n_cand for c in real)
        assert len(set(real)) == len(real)


def test_selection_is_the_best_biased_subset():
    # brute force: the selected set maximises the sum of biased group scores over the candidates
    # before the window (ties cannot occur with continuous random values)
    C, k, wc, T, d = 4, 2, 2, 36, 6
    Q, K, V, L = _problem(13, 1, 2, 1, T, d, C)
    bias = np.random.default_rng(14).standard_normal((1, 1, T // C)) * 2.0
    scale = 1.0 / math.sqrt(d)
    res = orc.forward_window(Q, K, V, L, C=C, k=k, wc=wc, scale=scale, bias=bias, nthreads=1)
    for i in range(0, T, 3):
        ci = i // C
        n_cand = max(ci - wc + 1, 0)
        qbar = Q[0, :, i, :].mean(axis=0)
        shat = [scale * float(qbar @ L[0, 0, c]) + float(bias[0, 0, c]) for c in range(n_cand)]
        m = min(k, n_cand)
        best = max(itertools.combinations(range(n_cand), m), key=lambda s: sum(shat[c] for c in s)) if m else ()
        got = sorted(int(c) for c in res["sel"][0, 0, i, :k] if c >= 0)
        assert got == sorted(best), (i, got, best)


def test_common_bias_changes_nothing_and_a_large_bias_is_retrieved_first():
    C, k, wc, T = 8, 3, 2, 160
    Q, K, V, L = _problem(17, 1, 2, 1, T, 8, C)
    nL = T // C
    base = orc.forward_window(Q, K, V, L, C=C, k=k, wc=wc, nthreads=2)
    shifted = orc.forward_window(Q, K, V, L, C=C, k=k, wc=wc, bias=np.full((1, 1, nL), 0.75), nthreads=2)
    assert np.array_equal(base["sel"], shifted["sel"])
    assert np.max(np.abs(base["w"] - shifted["w"])) <= 1e-12
    assert np.max(np.abs(base["O"] - shifted["O"])) <= 1e-12
    bias = np.zeros((1, 1, nL))
    bias[0, 0, 5] = 50.0
    res = orc.forward_window(Q, K, V, L, C=C, k=k, wc=wc, bias=bias, nthreads=2)
    for i in range(T):
        if i // C - wc + 1 > 5:        # chunk 5 is a retrieval candidate: it ranks first
            assert int(res["sel"][0, 0, i, 0]) == 5
            assert np.all(res["w"][0, :, i, 0] > 0.999)
        else:                          # chunk 5 is in the window or not visible: never retrieved
            assert 5 not in [int(c) for c in res["sel"][0, 0, i, :k]]


def test_weights_are_a_distribution_over_filled_slots():
    Q, K, V, L = _problem(19, 2, 4, 2, 150, 8, 16)
    bias = np.random.default_rng(20).standard_normal((2, 2, 150 // 16 + 1))
    res = orc.forward_window(Q, K, V, L, C=16, k=2, wc=3, bias=bias, nthreads=2)
    w, s = res["w"], res["s"]
    assert np.all(w >= 0) and np.max(np.abs(w.sum(axis=-1) - 1.0)) <= 1e-12
    assert np.all((w == 0) == np.isneginf(s))


def test_decode_equals_the_last_prefill_query():
    # one query at the last position of the cache gives the same result as the last query of the
    # full prefill (the window and the bias depend on the position only)
    B, H, Hkv, T, d, C = 1, 4, 2, 203, 8, 16
    Q, K, V, L = _problem(23, B, H, Hkv, T, d, C)
    bias = np.random.default_rng(24).standard_normal((B, Hkv, -(-T // C)))
    full = orc.forward_window(Q, K, V, L, C=C, k=3, wc=2, bias=bias, nthreads=2)
    one = orc.forward_window(Q[:, :, T - 1:T], K, V, L, C=C, k=3, wc=2, q_offset=T - 1, bias=bias, nthreads=1)
    assert np.array_equal(full["sel"][:, :, T - 1:T], one["sel"])
    assert np.max(np.abs(full["O"][:, :, T - 1:T] - one["O"])) <= 1e-15


PINS = [test_one_chunk_window_without_bias_is_the_method, test_window_covering_every_chunk_is_dense_causal_attention,
        test_window_only_is_sliding_window_attention, test_window_plus_full_retrieval_is_dense,
        test_window_and_retrieved_chunks_are_disjoint_and_ordered, test_selection_is_the_best_biased_subset,
        test_common_bias_changes_nothing_and_a_large_bias_is_retrieved_first,
        test_weights_are_a_distribution_over_filled_slots, test_decode_equals_the_last_prefill_query]

PLANTED = {
    12: "window taken one chunk early (own chunk left out)",
    13: "bias left out of the fusion weights",
    14: "window chunks also ranked as retrieval candidates",
}


def _broken_pins():
    broken = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            broken.append(pin.__name__)
    return broken


@pytest.mark.parametrize("m", sorted(PLANTED), ids=lambda m: "mistake%d" % m)
def test_planted_mistake_in_the_extension_is_caught(m):
    try:
        orc.set_mutant(m)
        broken = _broken_pins()
    finally:
        orc.set_mutant(0)
    assert broken, "planted mistake %d (%s) broke no pin" % (m, PLANTED[m])
