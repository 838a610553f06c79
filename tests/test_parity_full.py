"""GPU vs oracle at the full benchmark sizes, on sampled query groups (every (b, kv-head) group of
the decode workloads).

Inputs are generated on the device by the CUDA twin of the seeded generator, first checked to agree
bit for bit with the host generator on sampled elements of every tensor; the oracle then reads the rows
each sampled query group needs from those generated tensors (copied to the host and widened exactly to
float64), which spares the host generator the whole key cache behind every chunk-mean landmark.  The
library runs in the same launch configuration the benchmark times.
"""
import json

import numpy as np
import pytest
import torch

import parity
from oracle import oracle as orc
from synth import gpu as synth_gpu
from synth import workloads as W
from synth.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def raw_view(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    return t


def check_generator(w, dev, rng, n=256):
    """Sampled elements of every device tensor equal the host generator's raw values bit for bit."""
    shapes = {"Q": (w.B, w.H, w.N, w.d), "K": (w.B, w.Hkv, w.T, w.d), "V": (w.B, w.Hkv, w.T, w.d),
              "L": (w.B, w.Hkv, w.nL, w.d)}
    rows = {"Q": lambda b, x, r: W.q_rows(w, b, [x], np.array([r]))[1],
            "K": lambda b, x, r: W.k_rows(w, b, x, r, r + 1)[1],
            "V": lambda b, x, r: W.v_rows(w, b, x, r, r + 1)[1],
            "L": lambda b, x, r: W.l_rows(w, b, x, r, r + 1)[1]}
    for name, shp in shapes.items():
        idx = [rng.integers(0, s, size=n) for s in shp]
        flat = torch.from_numpy(np.ravel_multi_index(idx, shp)).cuda()
        got = raw_view(dev[name]).reshape(-1)[flat].cpu().numpy()
        want = [rows[name](int(idx[0][a]), int(idx[1][a]), int(idx[2][a])).reshape(-1)[int(idx[3][a])]
                for a in range(n)]
        if w.dtype == "bf16":
            assert np.array_equal(got.view(np.uint16), np.array(want, dtype=np.uint16)), name
        else:
            assert np.array_equal(got, np.array(want, dtype=np.float32)), name


def sample_items(w, rng, n_random):
    items = set()
    if w.N == 1:
        return [(b, g, 0) for b in range(w.B) for g in range(w.Hkv)]
    for _ in range(n_random):
        items.add((int(rng.integers(w.B)), int(rng.integers(w.Hkv)), int(rng.integers(w.N))))
    for i in (0, 1, w.C - 1, w.C, w.C * w.k, w.C * (w.k + 1) + 3, w.N - 1):
        if i < w.N:
            items.add((0, 0, i))
            items.add((w.B - 1, w.Hkv - 1, i))
    if w.n_needles:
        for i in range(0, w.N, w.needle_period * max(1, w.N // (w.needle_period * 48))):
            items.add((int(rng.integers(w.B)), int(rng.integers(w.Hkv)), i))
    return sorted(items)


def needle_recall(w, items, sel):
    """Fraction of needle queries whose selection holds at least one needle chunk of their group."""
    hits = tot = 0
    for (b, g, i), s in zip(items, sel):
        p = w.q_offset + i
        if not w.n_needles or p % w.needle_period:
            continue
        nc = set(int(c) for c in W.needle_chunks(w, g) if c < p // w.C)
        if not nc:
            continue
        tot += 1
        hits += bool(nc & set(int(c) for c in s))
    return hits / tot if tot else None


def answers_from_generated(w, dev, items, eps):
    """Oracle answers for items [(b, g, i)], reading the generated device tensors (float64 on the host);
    landmark rows are copied once per (b, g), key and value rows once per chunk."""
    scale = orc.default_scale(w.d)
    res = [None] * len(items)
    by_bg = {}
    for n, (b, g, i) in enumerate(items):
        by_bg.setdefault((int(b), int(g)), []).append((n, int(i)))
    for (b, g), lst in by_bg.items():
        ci_max = max((w.q_offset + i) // w.C for _, i in lst)
        Lrows = dev["L"][b, g, :ci_max + 1].double().cpu().numpy()
        cache = {}

        def fetch(c, b=b, g=g, cache=cache):
            if c not in cache:
                t0, t1 = c * w.C, min((c + 1) * w.C, w.T)
                cache[c] = (dev["K"][b, g, t0:t1].double().cpu().numpy(), dev["V"][b, g, t0:t1].double().cpu().numpy())
            return cache[c]

        heads = slice(g * w.G, (g + 1) * w.G)
        qi = torch.tensor([i for _, i in lst], device=dev["Q"].device)
        qs = dev["Q"][b, heads][:, qi].double().cpu().numpy()     # [G, n, d]
        for a, (n, i) in enumerate(lst):
            res[n] = orc.evaluate_query(qs[:, a, :], Lrows, fetch, w.C, w.k, w.q_offset + i, scale, eps)
    return res


@pytest.mark.parametrize("name,n_random", [("prefill_8k", 1024), ("prefill_256k_needles", 384),
                                           ("decode_128k", 0), ("decode_4m_needles", 0)])
def test_full_size(name, n_random):
    w = WORKLOADS[name]
    rng = np.random.default_rng(7)
    dev = synth_gpu.alloc_inputs(w)
    check_generator(w, dev, rng, n=256)
    O, sel_idx, sel_score = parity.gpu_run(w, dev, out_dtype="f32")
    items = sample_items(w, rng, n_random)
    sel, s, o = parity.gather_gpu(w, O, sel_idx, sel_score, items)
    del O, sel_idx, sel_score
    ans = answers_from_generated(w, dev, items, eps=parity.EPS_TIE)
    del dev
    torch.cuda.empty_cache()
    st = parity.compare(w, items, ans, sel, s, o)
    summary = {k: v for k, v in st.items() if k != "fail"}
    summary["needle_recall"] = needle_recall(w, items, sel)
    print("FULLSIZE", name, json.dumps(summary))
    assert st["fail"] == [], st["fail"][:5]
