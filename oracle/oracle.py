"""ctypes wrapper of the float64 CPU oracle (``oracle/hils_oracle.c``).

TEST INFRASTRUCTURE: imported only by the tests, the smoke check and the CPU
baseline leg of the benchmark.  The product library never imports it.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hils_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libhils_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def build(force=False):
    """Compile the oracle with gcc (IEEE float64: no fast-math, no contraction)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fPIC",
                           "-shared", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        L.hils_oracle_set_mutant.argtypes = [ctypes.c_int]
        L.hils_oracle_group_scores.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, _D, _D]
        L.hils_oracle_topk.argtypes = [ctypes.c_int, ctypes.c_int, _D, _I]
        L.hils_oracle_topk.restype = ctypes.c_int
        L.hils_oracle_select.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                         ctypes.c_double, _D, _D, _I, _D]
        L.hils_oracle_attend.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                         ctypes.c_double, _D, _I, _D, _D, _D, _D, _D, _D, _D]
        L.hils_oracle_tie_alternatives.argtypes = [ctypes.c_int, ctypes.c_int, _D, ctypes.c_double, ctypes.c_int, _I]
        L.hils_oracle_tie_alternatives.restype = ctypes.c_int
        L.hils_oracle_forward.argtypes = [ctypes.c_int] * 8 + [ctypes.c_long, ctypes.c_double, _D, _D, _D, _D,
                                                               _D, _I, _D, _D, ctypes.c_int]
        L.hils_oracle_forward.restype = ctypes.c_int
        L.hils_oracle_forward_window.argtypes = [ctypes.c_int] * 9 + [ctypes.c_long, ctypes.c_double, _D, _D, _D,
                                                                      _D, _D, _D, _I, _D, _D, ctypes.c_int]
        L.hils_oracle_forward_window.restype = ctypes.c_int
        L.hils_oracle_landmarks.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, _D, _D, _D]
        L.hils_oracle_select_window.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_long, ctypes.c_double, _D, _D, _D, _I, _D]
        L.hils_oracle_attend_slots.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_long,
                                               ctypes.c_double, _D, _I, _D, _D, _D, _D, _D, _D, _D]
        L.hils_oracle_max_threads.restype = ctypes.c_int
    return _lib


def _dp(a):
    return a.ctypes.data_as(_D) if a is not None else None


def _ip(a):
    return a.ctypes.data_as(_I) if a is not None else None


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def set_mutant(m):
    lib().hils_oracle_set_mutant(int(m))


def max_threads():
    return lib().hils_oracle_max_threads()


def default_scale(d):
    return 1.0 / np.sqrt(d)


def forward(Q, K, V, L, C, k, q_offset=0, scale=None, nthreads=None):
    """Whole forward pass.  Q [B,H,N,d], K/V [B,Hkv,T,d], L [B,Hkv,ceil(T/C),d] (float64).

    Returns dict with O [B,H,N,d], sel [B,Hkv,N,k+1], s and w [B,H,N,k+1].
    """
    Q, K, V, L = _f64(Q), _f64(K), _f64(V), _f64(L)
    B, H, N, d = Q.shape
    _, Hkv, T, _ = K.shape
    assert L.shape == (B, Hkv, -(-T // C), d), L.shape
    scale = default_scale(d) if scale is None else scale
    O = np.zeros((B, H, N, d))
    sel = np.zeros((B, Hkv, N, k + 1), dtype=np.int32)
    s = np.zeros((B, H, N, k + 1))
    w = np.zeros((B, H, N, k + 1))
    nthreads = max_threads() if nthreads is None else nthreads
    rc = lib().hils_oracle_forward(B, H, Hkv, N, T, d, C, k, q_offset, scale, _dp(Q), _dp(K), _dp(V), _dp(L),
                                   _dp(O), _ip(sel), _dp(s), _dp(w), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the shapes")
    return {"O": O, "sel": sel, "s": s, "w": w}


def forward_window(Q, K, V, L, C, k, wc, q_offset=0, scale=None, bias=None, nthreads=None):
    """Forward pass with a local window of wc chunks (the own chunk and the wc-1 before it, always
    attended; retrieval ranks only the chunks before the window) and an optional per-chunk bias
    [B,Hkv,ceil(T/C)] added to the retrieval scores.  wc = 1 and bias None give forward().

    Returns dict with O [B,H,N,d], sel [B,Hkv,N,k+wc] (top-k in rank order, then the window
    chunks ascending), s and w [B,H,N,k+wc].
    """
    Q, K, V, L = _f64(Q), _f64(K), _f64(V), _f64(L)
    B, H, N, d = Q.shape
    _, Hkv, T, _ = K.shape
    nL = -(-T // C)
    assert L.shape == (B, Hkv, nL, d), L.shape
    if bias is not None:
        bias = _f64(bias)
        assert bias.shape == (B, Hkv, nL), bias.shape
    scale = default_scale(d) if scale is None else scale
    ns = k + wc
    O = np.zeros((B, H, N, d))
    sel = np.zeros((B, Hkv, N, ns), dtype=np.int32)
    s = np.zeros((B, H, N, ns))
    w = np.zeros((B, H, N, ns))
    nthreads = max_threads() if nthreads is None else nthreads
    rc = lib().hils_oracle_forward_window(B, H, Hkv, N, T, d, C, k, wc, q_offset, scale, _dp(Q), _dp(K), _dp(V),
                                          _dp(L), _dp(bias) if bias is not None else None, _dp(O), _ip(sel),
                                          _dp(s), _dp(w), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the shapes")
    return {"O": O, "sel": sel, "s": s, "w": w}


def landmarks(K, U, C, scale=None):
    """Landmarks L [B,Hkv,nL,d] and entropy biases beta [B,Hkv,nL] from keys K [B,Hkv,T,d] and
    per-chunk landmark queries U [B,Hkv,nL,d]: L_c = sum_t p_t k_t, beta_c = -sum_t p_t log p_t,
    p = softmax over the chunk's keys of scale * u_c . k_t."""
    K, U = _f64(K), _f64(U)
    B, Hkv, T, d = K.shape
    nL = -(-T // C)
    assert U.shape == (B, Hkv, nL, d), U.shape
    scale = default_scale(d) if scale is None else scale
    L = np.zeros((B, Hkv, nL, d))
    beta = np.zeros((B, Hkv, nL))
    for b in range(B):
        for g in range(Hkv):
            Lbg = np.zeros((nL, d))
            bbg = np.zeros(nL)
            lib().hils_oracle_landmarks(T, d, C, scale, _dp(np.ascontiguousarray(K[b, g])),
                                        _dp(np.ascontiguousarray(U[b, g])), _dp(Lbg), _dp(bbg))
            L[b, g], beta[b, g] = Lbg, bbg
    return L, beta


def group_scores(q, Lrows, scale):
    q, Lrows = _f64(q), _f64(Lrows)
    G, d = q.shape
    out = np.zeros(Lrows.shape[0])
    lib().hils_oracle_group_scores(G, d, Lrows.shape[0], scale, _dp(q), _dp(Lrows), _dp(out))
    return out


def topk(shat, n_past, k):
    shat = _f64(shat)
    sel = np.zeros(max(k, 1), dtype=np.int32)
    lib().hils_oracle_topk(n_past, k, _dp(shat), _ip(sel))
    return sel[:k]


def select(q, Lrows, C, k, pos, scale):
    """q [G,d]; Lrows [>= pos//C + 1, d] landmarks from chunk 0.  Returns (sel[k+1], shat[c_i+1])."""
    q = _f64(q)
    G, d = q.shape
    ci = pos // C
    Lrows = _f64(Lrows[:ci + 1])
    sel = np.zeros(k + 1, dtype=np.int32)
    shat = np.zeros(ci + 1)
    lib().hils_oracle_select(G, d, C, k, pos, scale, _dp(q), _dp(Lrows), _ip(sel), _dp(shat))
    return sel, shat


def attend(q, sel, Lsel, Ksel, Vsel, C, pos, scale, want_chunks=False):
    """q [G,d]; sel [k+1]; Lsel [k+1,d]; Ksel/Vsel [k+1,C,d].  Returns dict s, w [G,k+1], o [G,d] (+ oc)."""
    q = _f64(q)
    G, d = q.shape
    ns = len(sel)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    Lsel, Ksel, Vsel = _f64(Lsel), _f64(Ksel), _f64(Vsel)
    assert Ksel.shape == (ns, C, d) and Vsel.shape == (ns, C, d) and Lsel.shape == (ns, d)
    s = np.zeros((G, ns))
    w = np.zeros((G, ns))
    o = np.zeros((G, d))
    oc = np.zeros((G, ns, d)) if want_chunks else None
    lib().hils_oracle_attend(G, d, C, ns - 1, pos, scale, _dp(q), _ip(sel), _dp(Lsel), _dp(Ksel), _dp(Vsel),
                             _dp(s), _dp(w), _dp(o), _dp(oc))
    out = {"s": s, "w": w, "o": o}
    if want_chunks:
        out["oc"] = oc
    return out


def attend_slots(q, sel, Lsel, bsel, Ksel, Vsel, C, pos, scale):
    """Attention inside the given slots and their fusion, for one query group (the windowed form).

    q [G,d]; sel [ns] chunk per slot (-1 empty); Lsel [ns,d]; bsel [ns] slot biases or None;
    Ksel/Vsel [ns,C,d].  Returns dict s, w [G,ns], o [G,d] with s = scale q.L_c + bias_c."""
    q = _f64(q)
    G, d = q.shape
    ns = len(sel)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    Lsel, Ksel, Vsel = _f64(Lsel), _f64(Ksel), _f64(Vsel)
    assert Ksel.shape == (ns, C, d) and Vsel.shape == (ns, C, d) and Lsel.shape == (ns, d)
    bsel = _f64(bsel) if bsel is not None else None
    s = np.zeros((G, ns))
    w = np.zeros((G, ns))
    o = np.zeros((G, d))
    lib().hils_oracle_attend_slots(G, d, C, ns, pos, scale, _dp(q), _ip(sel), _dp(Lsel), _dp(bsel), _dp(Ksel),
                                   _dp(Vsel), _dp(s), _dp(w), _dp(o))
    return {"s": s, "w": w, "o": o}


def tie_alternatives(shat, n_past, k, eps, max_alts=64):
    """Alternative top-k selections within the near-tie band (first = primary); None if too many."""
    shat = _f64(shat)
    alts = np.zeros((max_alts, max(k, 1)), dtype=np.int32)
    n = lib().hils_oracle_tie_alternatives(n_past, k, _dp(shat), eps, max_alts, _ip(alts))
    if n < 0:
        return None
    return [alts[a, :k].copy() for a in range(n)]


# ---------------------------------------------------------------------------
# One query group at a time, for sampled comparisons on large inputs.

def evaluate_query(q, Lrows, fetch_kv, C, k, pos, scale, eps=1e-3, max_alts=16):
    """Oracle answer for one query group.

    q [G,d]; Lrows [>= c_i+1, d] landmarks from chunk 0; fetch_kv(c) -> (K rows, V rows)
    of chunk c (at most C rows each).  Returns dict: shat (group scores of chunks
    0..c_i), overflow (near-tie band too large to enumerate), alts: list of
    (sel[k+1], s[G,k+1], w[G,k+1], o[G,d]), the primary selection first and then
    every other selection a near tie (score gap <= eps) would allow.
    """
    q = _f64(q)
    G, d = q.shape
    ci = pos // C
    sel, shat = select(q, Lrows, C, k, pos, scale)
    alts = tie_alternatives(shat, ci, k, eps, max_alts)
    overflow = alts is None
    if overflow:
        alts = [sel[:k]]
    cache = {}
    out = []
    for a in alts:
        full = np.concatenate([a, [ci]]).astype(np.int32)
        Ls = np.zeros((k + 1, d))
        Ks = np.zeros((k + 1, C, d))
        Vs = np.zeros((k + 1, C, d))
        for j, c in enumerate(full):
            c = int(c)
            if c < 0:
                continue
            if c not in cache:
                cache[c] = fetch_kv(c)
            kk, vv = cache[c]
            Ls[j] = Lrows[c]
            Ks[j, :kk.shape[0]] = kk
            Vs[j, :vv.shape[0]] = vv
        r = attend(q, full, Ls, Ks, Vs, C, pos, scale)
        out.append((full, r["s"], r["w"], r["o"]))
    return {"pos": pos, "shat": shat, "alts": out, "overflow": overflow}


def sample_queries(w, items, eps=1e-3, max_alts=16):
    """Oracle answers for query groups items = [(b, g, i), ...] of a synth Workload.

    Inputs are rebuilt from the seeded generator, slice by slice; landmarks are
    generated once per (b, g).
    """
    from synth import workloads as W
    scale = default_scale(w.d)
    res = [None] * len(items)
    by_bg = {}
    for n, (b, g, i) in enumerate(items):
        by_bg.setdefault((int(b), int(g)), []).append((n, int(i)))
    for (b, g), lst in by_bg.items():
        ci_max = max((w.q_offset + i) // w.C for _, i in lst)
        Lrows, _ = W.l_rows(w, b, g, 0, ci_max + 1)
        heads = np.arange(g * w.G, (g + 1) * w.G)
        kv_cache = {}

        def fetch(c, b=b, g=g, kv_cache=kv_cache):
            if c not in kv_cache:
                t0, t1 = c * w.C, min((c + 1) * w.C, w.T)
                kv_cache[c] = (W.k_rows(w, b, g, t0, t1)[0], W.v_rows(w, b, g, t0, t1)[0])
            return kv_cache[c]

        qs, _ = W.q_rows(w, b, heads, np.array([i for _, i in lst]))
        for a, (n, i) in enumerate(lst):
            res[n] = evaluate_query(qs[:, a, :], Lrows, fetch, w.C, w.k, w.q_offset + i, scale, eps, max_alts)
    return res
