"""Local window and per-chunk bias on the GPU (hils_score_select_window, hils_forward_window) against the
oracle's extension of the method (oracle.forward_window).

The window is the own chunk and the wc - 1 chunks before it, attended and fused like retrieved chunks;
retrieval ranks only the chunks before the window, by the group score plus the chunk's bias, and the
bias also enters every slot's fusion score ("Hierarchical Sparse Attention Done Right", Sec. 2
Preliminary and Sec. 5 "Experimental setup" for the window, Sec. 3 "Linear surrogate for chunk mass"
for the bias).  Checks per query group: the window slots exactly; the retrieved chunks exactly in rank
order unless the oracle's k-th and (k+1)-th biased group scores lie within 1e-3 (such near ties are
counted and left out); slot scores within 1e-4; outputs within 1e-4 (float32 inputs) or 1e-2 (bf16).
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


def _near_ties(w, wc, arr, bias):
    """[B, Hkv, N] bool: the oracle's k-th and (k+1)-th biased group scores lie within EPS_TIE."""
    scale = 1.0 / math.sqrt(w.d)
    out = np.zeros((w.B, w.Hkv, w.N), dtype=bool)
    for b in range(w.B):
        for g in range(w.Hkv):
            for i in range(w.N):
                n_cand = (w.q_offset + i) // w.C - wc + 1
                if n_cand <= w.k or w.k == 0:
                    continue
                q = arr["Q"][b, g * w.G:(g + 1) * w.G, i]
                gs = orc.group_scores(q, arr["L"][b, g, :n_cand], scale)
                if bias is not None:
                    gs = gs + bias[b, g, :n_cand].astype(np.float64)
                gs = np.sort(gs)[::-1]
                out[b, g, i] = gs[w.k - 1] - gs[w.k] < EPS_TIE
    return out


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_window_and_bias_match_the_oracle(case):
    w, wc, bias_scale = case
    arr, bias, ref, sel, s, O = _run(w, wc, bias_scale)
    kp = w.k + wc - 1
    tie = _near_ties(w, wc, arr, bias)
    assert tie.mean() < 0.2, tie.mean()
    # window slots: exact for every query group
    assert np.array_equal(sel[..., w.k:], ref["sel"][..., w.k:kp])
    keep_g = ~tie
    assert np.array_equal(sel[..., :w.k][keep_g], ref["sel"][..., :w.k][keep_g])
    keep_h = np.repeat(keep_g, w.G, axis=1)
    rs = ref["s"][keep_h]
    gs = s[keep_h]
    assert np.array_equal(np.isneginf(gs), np.isneginf(rs))
    fin = ~np.isneginf(rs)
    assert np.max(np.abs(gs[fin] - rs[fin]), initial=0.0) <= TOL_S
    tol = 1e-4 if w.dtype == "f32" else 1e-2
    err = np.max(np.abs(O[keep_h] - ref["O"][keep_h]), initial=0.0)
    assert err <= tol, err
