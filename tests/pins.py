"""Pins of the float64 oracle against facts that do not come from the oracle.

Each ``pin_*`` function returns a list of failure strings (empty = pinned).
They are shared by ``test_oracle_pins.py`` (every pin must hold) and
``test_oracle_mutants.py`` (every planted mistake must break at least one pin).

What pins what:
  * dense reduction: chunk size 1, landmarks = keys, k >= #chunks => the output is
    plain causal softmax attention (torch's scaled_dot_product_attention, float64).
  * one chunk: N = T = C => causal softmax attention, for any landmarks and k.
  * hand-derived worked example (tests/golden/hand_worked_d2.json).
  * brute-force selection: maximum-sum k-subset, lexicographically smallest on ties.
  * planted exact ties (duplicate landmarks) go to the lower chunk index.
  * planted needle: a landmark aligned with the query is retrieved.
  * invariances: common landmark shift, per-chunk key shift, constant values,
    causality (future rows do not matter), decode == last prefill query,
    identical heads == one head.
  * fusion weights are a distribution over the filled slots.
  * matrix form: given only the selected chunk indices, a dense attention row
    A_ij = w_{c(j)} * softmax over chunk c(j)'s visible keys, with the weights recomputed
    here from the landmark scores, reproduces the output (o = A V); its rows sum to 1 and
    it is zero outside the selected chunks' visible ranges.
"""
import itertools
import json
import math
import os

import numpy as np
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _problem(seed, B, H, Hkv, T, d, C, l_equals_k=False):
    r = _rng(seed)
    Q = r.standard_normal((B, H, T, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    nL = -(-T // C)
    L = K.copy() if l_equals_k else r.standard_normal((B, Hkv, nL, d))
    return Q, K, V, L


def _sdpa_causal(Q, K, V, scale):
    G = Q.shape[1] // K.shape[1]
    q = torch.from_numpy(Q)
    k = torch.from_numpy(K).repeat_interleave(G, dim=1)
    v = torch.from_numpy(V).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale).numpy()


def _maxerr(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    if a.shape != b.shape:
        return math.inf
    with np.errstate(invalid="ignore"):
        e = np.abs(a - b)
    return float(np.nanmax(e)) if not np.isnan(e).any() else math.inf


def pin_dense_reduction():
    fails = []
    for (B, H, Hkv, T, d) in [(2, 4, 2, 40, 16), (1, 3, 3, 33, 8)]:
        Q, K, V, L = _problem(11 + T, B, H, Hkv, T, d, 1, l_equals_k=True)
        scale = 1.0 / math.sqrt(d)
        res = orc.forward(Q, K, V, L, C=1, k=T, scale=scale, nthreads=2)
        ref = _sdpa_causal(Q, K, V, scale)
        e = _maxerr(res["O"], ref)
        if not e <= 1e-12:
            fails.append("dense reduction B%d H%d Hkv%d T%d d%d: max err %.3g" % (B, H, Hkv, T, d, e))
    return fails


def pin_one_chunk():
    fails = []
    for (C, k) in [(16, 0), (16, 3)]:
        Q, K, V, L = _problem(5 + k, 1, 2, 1, C, 8, C)
        scale = 1.0 / math.sqrt(8)
        res = orc.forward(Q, K, V, L, C=C, k=k, scale=scale, nthreads=1)
        ref = _sdpa_causal(Q, K, V, scale)
        e = _maxerr(res["O"], ref)
        if not e <= 1e-12:
            fails.append("one chunk C%d k%d: max err %.3g" % (C, k, e))
    return fails


def _ln(v):
    if isinstance(v, str):
        return math.log(float(v[2:]))
    return float(v)


def pin_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_d2.json")))
    T, d, C, k = 6, 2, 2, 1
    Q = np.zeros((1, 1, T, d))
    Q[0, 0, :, 0] = [_ln(x) for x in g["Q_first"]]
    K = np.zeros((1, 1, T, d))
    K[0, 0, :, 0] = [_ln(x) for x in g["K_first"]]
    K[0, 0, :, 1] = g["K_second"]
    V = np.array(g["V"], dtype=np.float64).reshape(1, 1, T, d)
    L = np.zeros((1, 1, 3, d))
    L[0, 0, :, 0] = [_ln(x) for x in g["L_first"]]
    L[0, 0, :, 1] = g["L_second"]
    res = orc.forward(Q, K, V, L, C=C, k=k, scale=1.0, nthreads=1)
    fails = []
    if not np.array_equal(res["sel"][0, 0], np.array(g["expected_sel"])):
        fails.append("hand example: selection %s" % res["sel"][0, 0].tolist())
    e = _maxerr(res["O"][0, 0], np.array(g["expected_O"]))
    if not e <= 1e-13:
        fails.append("hand example: output err %.3g" % e)
    e = _maxerr(res["w"][0, 0], np.array(g["expected_w"]))
    if not e <= 1e-15:
        fails.append("hand example: weight err %.3g" % e)
    return fails


def pin_brute_force_selection():
    """Top-k against enumeration of every k-subset of the past chunks (tiny inputs)."""
    fails = []
    r = _rng(3)
    for trial in range(40):
        G = 1 + trial % 3
        d = 4
        n_chunks = 2 + trial % 9          # chunks 0..n_chunks-1, query in the last one
        C = 1 + trial % 3
        k = trial % 5
        # integer-valued landmarks/queries make exact score ties frequent
        q = r.integers(-2, 3, size=(G, d)).astype(np.float64)
        Lr = r.integers(-2, 3, size=(n_chunks, d)).astype(np.float64)
        pos = (n_chunks - 1) * C + (trial % C)
        sel, shat = orc.select(q, Lr, C, k, pos, 0.5)
        ci = pos // C
        # independent group score: per-head dot products summed in numpy, divided by G
        ref_shat = np.array([sum(0.5 * float(np.dot(q[h], Lr[c])) for h in range(G)) / G for c in range(ci + 1)])
        if _maxerr(shat, ref_shat) > 1e-12:
            fails.append("group scores differ from the per-head mean (trial %d)" % trial)
        m = min(k, ci)
        best = None
        for sub in itertools.combinations(range(ci), m):
            key = (-sum(ref_shat[list(sub)]), sub)
            if best is None or key < best:
                best = key
        want = sorted(best[1]) if best else []
        got = sel[:k]
        if sorted(int(x) for x in got if x >= 0) != want or int(sel[k]) != ci or (got < 0).sum() != k - m:
            fails.append("brute force trial %d: got %s want %s" % (trial, sel.tolist(), want))
        # rank order: by score descending, ties by index ascending
        ranked = [int(x) for x in got if x >= 0]
        if ranked != sorted(ranked, key=lambda c: (-ref_shat[c], c)):
            fails.append("rank order trial %d: %s" % (trial, ranked))
    return fails


def pin_tie_lowest_index():
    fails = []
    d = 8
    r = _rng(9)
    q = r.standard_normal((2, d))
    Lr = r.standard_normal((12, d)) * 0.1
    Lr[3] = Lr[7] = Lr[10] = q.mean(axis=0) * 5      # three exact duplicates, the best score
    sel, _ = orc.select(q, Lr, 4, 2, 11 * 4 + 1, 0.3)
    if sel[:2].tolist() != [3, 7]:
        fails.append("ties: got %s want [3, 7]" % sel[:2].tolist())
    return fails


def pin_needle_retrieved():
    fails = []
    d, C = 16, 8
    r = _rng(21)
    q = r.standard_normal((4, d))
    for needle in (0, 5, 30):
        Lr = r.standard_normal((40, d))
        Lr[needle] = q.mean(axis=0) * 20.0
        sel, _ = orc.select(q, Lr, C, 3, 39 * C + 2, 1.0 / math.sqrt(d))
        if int(sel[0]) != needle:
            fails.append("needle %d not retrieved first: %s" % (needle, sel.tolist()))
    return fails


def pin_invariances():
    fails = []
    B, H, Hkv, T, d, C, k = 1, 4, 2, 48, 8, 4, 3
    Q, K, V, L = _problem(7, B, H, Hkv, T, d, C)
    base = orc.forward(Q, K, V, L, C=C, k=k, nthreads=2)
    # common landmark shift
    a = _rng(1).standard_normal(d)
    r1 = orc.forward(Q, K, V, L + a, C=C, k=k, nthreads=2)
    if not np.array_equal(r1["sel"], base["sel"]) or _maxerr(r1["O"], base["O"]) > 1e-12:
        fails.append("common landmark shift changed the result")
    # per-chunk key shift
    K2 = K.copy()
    K2[:, :, 2 * C:3 * C, :] += _rng(2).standard_normal(d)
    r2 = orc.forward(Q, K2, V, L, C=C, k=k, nthreads=2)
    if _maxerr(r2["O"], base["O"]) > 1e-12:
        fails.append("key shift inside one chunk changed the output")
    # constant values
    vconst = _rng(4).standard_normal(d)
    V3 = np.broadcast_to(vconst, V.shape).copy()
    r3 = orc.forward(Q, K, V3, L, C=C, k=k, nthreads=2)
    if _maxerr(r3["O"], np.broadcast_to(vconst, r3["O"].shape)) > 1e-13:
        fails.append("constant values not reproduced")
    # weights: distribution over filled slots
    w = base["w"]
    if _maxerr(w.sum(axis=-1), np.ones(w.shape[:-1])) > 1e-13 or (w < 0).any():
        fails.append("fusion weights do not form a distribution")
    G = H // Hkv
    empty = np.repeat(base["sel"] < 0, G, axis=1)
    if (w[empty] != 0).any():
        fails.append("empty slot with a non-zero weight")
    # causality: rows after position p do not change output p
    p = 29
    K4, V4, L4 = K.copy(), V.copy(), L.copy()
    K4[:, :, p + 1:] = 99.0
    V4[:, :, p + 1:] = -99.0
    L4[:, :, p // C + 1:] = 7.0
    r4 = orc.forward(Q, K4, V4, L4, C=C, k=k, nthreads=2)
    if _maxerr(r4["O"][:, :, :p + 1], base["O"][:, :, :p + 1]) > 1e-13:
        fails.append("future rows changed a past output")
    # decode of position p over a cache of length p+1 == prefill query p
    Tn = p + 1
    rd = orc.forward(Q[:, :, p:p + 1], K[:, :, :Tn], V[:, :, :Tn], L[:, :, :-(-Tn // C)], C=C, k=k,
                     q_offset=p, nthreads=1)
    if _maxerr(rd["O"][:, :, 0], base["O"][:, :, p]) > 1e-13:
        fails.append("decode differs from the prefill query at the same position")
    # identical heads in a group == one head
    Qi = np.repeat(Q[:, ::G], G, axis=1)
    ri = orc.forward(Qi, K, V, L, C=C, k=k, nthreads=2)
    r1h = orc.forward(Q[:, ::G], K, V, L, C=C, k=k, nthreads=2)
    if _maxerr(ri["O"], np.repeat(r1h["O"], G, axis=1)) > 1e-13:
        fails.append("identical heads differ from a single head")
    return fails


def pin_matrix_form():
    """The second, independent formulation of steps 3-6: one dense row of attention weights per
    (b, h, i) over all T keys, built with numpy from the selection alone."""
    fails = []
    for (B, H, Hkv, T, d, C, k, q_offset) in [(2, 4, 2, 70, 8, 8, 3, 0), (1, 2, 1, 100, 6, 16, 2, 60)]:
        N = T - q_offset
        Q, K, V, L = _problem(31 + T, B, H, Hkv, T, d, C)
        Q = Q[:, :, q_offset:]
        scale = 1.0 / math.sqrt(d)
        res = orc.forward(Q, K, V, L, C=C, k=k, q_offset=q_offset, scale=scale, nthreads=2)
        G = H // Hkv
        A = np.zeros((B, H, N, T))
        for b in range(B):
            for h in range(H):
                g = h // G
                for i in range(N):
                    pos = q_offset + i
                    chunks = [int(c) for c in res["sel"][b, g, i] if c >= 0]
                    if pos // C not in chunks or len(set(chunks)) != len(chunks):
                        fails.append("matrix form: slot list of (%d, %d, %d) is not past chunks + own" % (b, g, i))
                        continue
                    q = Q[b, h, i]
                    s = np.array([scale * q @ L[b, g, c] for c in chunks])
                    w = np.exp(s - s.max())
                    w /= w.sum()
                    for wc, c in zip(w, chunks):
                        j0, j1 = c * C, min(c * C + C, pos + 1)
                        logit = scale * K[b, g, j0:j1] @ q
                        p = np.exp(logit - logit.max())
                        A[b, h, i, j0:j1] = wc * p / p.sum()
        O = np.einsum("bhit,bhtd->bhid", A, np.repeat(V, G, axis=1))
        e = _maxerr(res["O"], O)
        if not e <= 1e-12:
            fails.append("matrix form B%d T%d q_offset %d: max err %.3g" % (B, T, q_offset, e))
        if _maxerr(A.sum(axis=-1), np.ones(A.shape[:-1])) > 1e-12:
            fails.append("matrix form: rows do not sum to 1")
        future = np.arange(T)[None, None, None, :] > (q_offset + np.arange(N))[None, None, :, None]
        if (A[np.broadcast_to(future, A.shape)] != 0).any():
            fails.append("matrix form: weight on a future key")
    return fails


ALL_PINS = [pin_dense_reduction, pin_one_chunk, pin_hand_worked, pin_brute_force_selection,
            pin_tie_lowest_index, pin_needle_retrieved, pin_invariances, pin_matrix_form]


def run_all():
    out = {}
    for p in ALL_PINS:
        try:
            out[p.__name__] = p()
        except Exception as e:  # a planted mistake may also crash a pin
            out[p.__name__] = ["raised %r" % (e,)]
    return out
