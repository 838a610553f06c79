"""Local window and per-chunk bias on the GPU (hils_score_select_window, hils_forward_window) against the
oracle's extension of the method (oracle.forward_window).

The window is the own chunk and the wc - 1 chunks before it, attended and fused like retrieved chunks;
retrieval ranks only the chunks before the window, by the group score plus the chunk's bias, and the
bias also enters every slot's fusion score ("Hierarchical Sparse Attention Done Right", Sec. 2
Preliminary and Sec. 5 "Experimental setup" for the window, Sec. 3 "Linear surrogate for chunk mass"
for the bias).  Checks per query group: the window slots exactly; the same retrieved chunks as the
oracle, ranked in an order its scores allow (two chunks may swap only within the 1e-3 near-tie band),
unless its k-th and (k+1)-th biased group scores lie within 1e-3 (such near ties at the cut are counted
and left out); every slot's score, matched by chunk, within 1e-4; outputs within 1e-4 (float32 inputs)
or 1e-2 (bf16).
"""
import math

import numpy as np
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
import parity
from oracle import oracle as orc
from synth import workloads as W
from synth.workloads import Workload

pytestmark = pytest.mark.gpu

EPS_TIE = 1e-3
TOL_S = 1e-4


def wl(name, **kw):
    base = dict(B=1, H=8, Hkv=2, N=1000, T=1000, d=128, C=64, k=4, q_offset=0, dtype="bf16", seed=150,
                l_mode="chunkmean")
    base.update(kw)
    return Workload(name, **base)


CASES = [
    # workload, window chunks, bias scale (None: no bias)
    (wl("prefill_bf16_g4_wc3_bias"), 3, 1.0),
    (wl("prefill_bf16_wc1_no_bias", seed=151), 1, None),
    (wl("prefill_f32_d64_c32_wc2", B=2, H=4, N=700, T=700, d=64, C=32, k=3, dtype="f32", seed=152,
        l_mode="iid"), 2, None),
    (wl("prefill_chunked_offset_wc4_bias", N=300, T=2000, q_offset=1700, k=6, seed=153), 4, 0.5),
    (wl("decode_bf16_g4_wc4_bias", B=2, N=1, T=5000, q_offset=4999, k=8, seed=154), 4, 1.0),
    (wl("decode_f32_window_past_the_start", B=2, H=4, Hkv=1, N=1, T=100, q_offset=99, d=64, C=32, k=2,
        dtype="f32", seed=155, l_mode="iid"), 8, 1.0),
    (wl("decode_long_wc8_bias", B=1, N=1, T=64 * 3000 + 5, q_offset=64 * 3000 + 4, k=16, seed=156,
        l_mode="iid"), 8, 2.0),
]


def _run(w, wc, bias_scale):
    inp = W.full_inputs(w)
    arr = {k: v[0] for k, v in inp.items()}
    dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
    bias = None
    if bias_scale is not None:
        bias = (np.random.default_rng(w.seed + 7).standard_normal((w.B, w.Hkv, w.nL)) * bias_scale).astype(np.float32)
    p = parity.problem_of(w)
    kp = w.k + wc - 1
    bias_d = torch.from_numpy(bias).cuda() if bias is not None else None
    sel_idx = torch.full((w.B, w.Hkv, w.N, max(kp, 1)), -7, dtype=torch.int32, device="cuda")
    sel_score = torch.empty((w.B, w.H, w.N, kp + 1), dtype=torch.float32, device="cuda")
    hils.hils_score_select_window(p, wc, bias_d, dev["Q"], dev["L"], sel_idx, sel_score)
    O = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    ws = torch.empty(hils.hils_forward_window_workspace_size(p, wc), dtype=torch.uint8, device="cuda")
    hils.hils_forward_window(p, wc, bias_d, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws)
    assert hils.hils_sync_status() == hils.HILS_OK
    ref = orc.forward_window(arr["Q"], arr["K"], arr["V"], arr["L"], w.C, w.k, wc, q_offset=w.q_offset,
                             bias=None if bias is None else bias.astype(np.float64))
    return arr, bias, ref, sel_idx[..., :kp].cpu().numpy(), sel_score.cpu().numpy(), O.double().cpu().numpy()


def _biased_group_scores(w, wc, arr, bias, b, g, i):
    """The oracle's biased group scores of query (b, g, i)'s candidates (float64)."""
    n_cand = max((w.q_offset + i) // w.C - wc + 1, 0)
    q = arr["Q"][b, g * w.G:(g + 1) * w.G, i]
    gs = orc.group_scores(q, arr["L"][b, g, :n_cand], 1.0 / math.sqrt(w.d)) if n_cand else np.zeros(0)
    if bias is not None and n_cand:
        gs = gs + bias[b, g, :n_cand].astype(np.float64)
    return gs


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_window_and_bias_match_the_oracle(case):
    w, wc, bias_scale = case
    arr, bias, ref, sel, s, O = _run(w, wc, bias_scale)
    kp = w.k + wc - 1
    # the window slots: exact for every query group
    assert np.array_equal(sel[..., w.k:], ref["sel"][..., w.k:kp])
    keep = np.ones((w.B, w.Hkv, w.N), dtype=bool)
    for b in range(w.B):
        for g in range(w.Hkv):
            for i in range(w.N):
                gs = _biased_group_scores(w, wc, arr, bias, b, g, i)
                order = np.sort(gs)[::-1]
                if w.k and len(gs) > w.k and order[w.k - 1] - order[w.k] < EPS_TIE:
                    keep[b, g, i] = False          # near tie at the cut: either chunk may be kept
                    continue
                got, want = sel[b, g, i, :w.k], ref["sel"][b, g, i, :w.k]
                assert sorted(got.tolist()) == sorted(want.tolist()), (b, g, i, got, want)
                real = [int(c) for c in got if c >= 0]
                # rank order: by the oracle's scores, up to the near-tie band
                assert all(gs[x] >= gs[y] - EPS_TIE for x, y in zip(real, real[1:])), (b, g, i, got)
                assert all(c == -1 for c in got[len(real):])
                # slot scores, matched by chunk (the window slots and the own chunk keep their places)
                for h in range(g * w.G, (g + 1) * w.G):
                    ref_by_chunk = {int(c): ref["s"][b, h, i, j] for j, c in enumerate(ref["sel"][b, g, i]) if c >= 0}
                    for j in range(kp + 1):
                        c = int(sel[b, g, i, j]) if j < kp else (w.q_offset + i) // w.C
                        if c < 0:
                            assert np.isneginf(s[b, h, i, j])
                        else:
                            assert abs(s[b, h, i, j] - ref_by_chunk[c]) <= TOL_S, (b, h, i, j)
    assert keep.mean() > 0.8, keep.mean()
    keep_h = np.repeat(keep, w.G, axis=1)
    tol = 1e-4 if w.dtype == "f32" else 1e-2
    err = np.max(np.abs(O[keep_h] - ref["O"][keep_h]), initial=0.0)
    assert err <= tol, err
