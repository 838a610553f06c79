"""Landmark generation on the GPU (hils_landmarks) against the oracle.

Per chunk, a landmark query attends over the chunk's own keys: the landmark is the attention-weighted
key sum and the bias the attention's entropy ("Hierarchical Sparse Attention Done Right", Sec. 3
Methodology, "Linear surrogate for chunk mass").  Both sides read the same inputs (bf16 inputs widened
exactly for the oracle).  Bounds: landmarks and biases within 1e-4 (float32 arithmetic against the
float64 oracle); a bf16 landmark is also allowed its own rounding to bf16 (half an ulp, at most
2^-8 of its magnitude).  Rows outside the requested chunk range must stay untouched.
"""
import math

import numpy as np
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

TOL = 1e-4
DEV = "cuda:0"


def _inputs(B, Hkv, T, d, C, dtype, seed, u_scale=1.0):
    r = np.random.default_rng(seed)
    nL = -(-T // C)
    K = torch.from_numpy(r.standard_normal((B, Hkv, T, d)).astype(np.float32))
    U = torch.from_numpy((r.standard_normal((B, Hkv, nL, d)) * u_scale).astype(np.float32))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    K, U = K.to(tdt), U.to(tdt)                       # round once; the oracle sees the rounded values
    return K, U, K.double().numpy(), U.double().numpy()


def _run(B, Hkv, T, d, C, dtype, seed, c_begin=0, c_end=None, u_scale=1.0, with_beta=True):
    K, U, K64, U64 = _inputs(B, Hkv, T, d, C, dtype, seed, u_scale)
    nL = -(-T // C)
    c_end = nL if c_end is None else c_end
    dt = hils.HILS_BF16 if dtype == "bf16" else hils.HILS_F32
    p = hils.problem(B, 1, Hkv, 1, T, d, C, 0, 0, dt)
    Kd, Ud = K.to(DEV), U.to(DEV)
    Ld = torch.full((B, Hkv, nL, d), float("nan"), dtype=K.dtype, device=DEV)
    bd = torch.full((B, Hkv, nL), float("nan"), dtype=torch.float32, device=DEV) if with_beta else None
    hils.hils_landmarks(p, Kd, Ud, Ld, bd, c_begin, c_end)
    assert hils.hils_sync_status() == hils.HILS_OK
    Lref, bref = orc.landmarks(K64, U64, C, scale=float(np.float32(1.0 / math.sqrt(d))))
    Lg = Ld.double().cpu().numpy()
    bg = bd.double().cpu().numpy() if with_beta else None
    return Lg, bg, Lref, bref, c_begin, c_end, dtype


def _check(Lg, bg, Lref, bref, c_begin, c_end, dtype):
    sl = slice(c_begin, c_end)
    bound = TOL + (2.0 ** -8) * np.abs(Lref[:, :, sl]) if dtype == "bf16" else TOL
    err = np.abs(Lg[:, :, sl] - Lref[:, :, sl])
    assert np.all(err <= bound), "landmark max error %.3g" % float(np.max(err))
    outside = np.delete(Lg, np.arange(c_begin, c_end), axis=2)
    assert np.all(np.isnan(outside)), "rows outside the chunk range were written"
    if bg is not None:
        eb = np.abs(bg[:, :, sl] - bref[:, :, sl])
        assert np.all(eb <= TOL), "bias max error %.3g" % float(np.max(eb))
        assert np.all(np.isnan(np.delete(bg, np.arange(c_begin, c_end), axis=2)))


CASES = [
    # name, B, Hkv, T, d, C, dtype, seed, extra
    ("bf16_d128_c64_ragged", 2, 4, 64 * 130 + 37, 128, 64, "bf16", 200, {}),
    ("bf16_d128_c128_peaky", 1, 2, 128 * 40, 128, 128, "bf16", 201, {"u_scale": 6.0}),
    ("bf16_d64_c32", 3, 2, 32 * 77 + 5, 64, 32, "bf16", 202, {}),
    ("f32_d64_c32_range", 2, 2, 32 * 50 + 9, 64, 32, "f32", 203, {"c_begin": 3, "c_end": 17}),
    ("f32_d128_c7", 1, 3, 7 * 60 + 3, 128, 7, "f32", 204, {}),
    ("f32_d64_c1", 1, 2, 75, 64, 1, "f32", 205, {}),
    ("f32_d128_last_chunk_only", 2, 2, 64 * 9 + 20, 128, 64, "f32", 206, {"c_begin": 9, "c_end": 10}),
    ("bf16_no_bias", 1, 2, 64 * 20, 128, 64, "bf16", 207, {"with_beta": False}),
    ("bf16_empty_range", 1, 1, 256, 128, 64, "bf16", 208, {"c_begin": 2, "c_end": 2}),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_landmarks_match_the_oracle(case):
    _, B, Hkv, T, d, C, dtype, seed, extra = case
    _check(*_run(B, Hkv, T, d, C, dtype, seed, **extra))


def test_landmarks_at_the_decode_cache_size():
    # the landmark cache of a 128K-token sequence (C = 64): 2,048 chunks per kv-head
    _check(*_run(1, 2, 131072, 128, 64, "bf16", 209))


def test_one_chunk_call_equals_the_same_chunk_of_a_full_call():
    # a decode step that completes a chunk recomputes only that chunk: same bits as the full pass
    B, Hkv, T, d, C = 2, 2, 64 * 12, 128, 64
    K, U, _, _ = _inputs(B, Hkv, T, d, C, "bf16", 210)
    p = hils.problem(B, 1, Hkv, 1, T, d, C, 0, 0, hils.HILS_BF16)
    Kd, Ud = K.to(DEV), U.to(DEV)
    full = torch.empty((B, Hkv, T // C, d), dtype=torch.bfloat16, device=DEV)
    fb = torch.empty((B, Hkv, T // C), dtype=torch.float32, device=DEV)
    hils.hils_landmarks(p, Kd, Ud, full, fb)
    one = torch.zeros_like(full)
    ob = torch.zeros_like(fb)
    for c in range(T // C):
        hils.hils_landmarks(p, Kd, Ud, one, ob, c, c + 1)
    assert hils.hils_sync_status() == hils.HILS_OK
    assert torch.equal(full.view(torch.int16), one.view(torch.int16))
    assert torch.equal(fb, ob)


def test_landmarks_feed_the_forward_pass():
    # landmarks produced on the GPU drive selection and attention; the oracle gets the same landmarks
    B, H, Hkv, T, d, C, k = 1, 4, 2, 64 * 16, 128, 64, 3
    K, U, _, _ = _inputs(B, Hkv, T, d, C, "bf16", 211)
    r = np.random.default_rng(212)
    Q = torch.from_numpy(r.standard_normal((B, H, T, d)).astype(np.float32)).to(torch.bfloat16)
    V = torch.from_numpy(r.standard_normal((B, Hkv, T, d)).astype(np.float32)).to(torch.bfloat16)
    p = hils.problem(B, H, Hkv, T, T, d, C, k, 0, hils.HILS_BF16, hils.HILS_F32)
    Kd, Ud, Qd, Vd = K.to(DEV), U.to(DEV), Q.to(DEV), V.to(DEV)
    Ld = torch.empty((B, Hkv, T // C, d), dtype=torch.bfloat16, device=DEV)
    hils.hils_landmarks(p, Kd, Ud, Ld)
    O = torch.empty((B, H, T, d), dtype=torch.float32, device=DEV)
    ws = torch.empty(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device=DEV)
    hils.hils_forward(p, Qd, Kd, Vd, Ld, O, ws)
    assert hils.hils_sync_status() == hils.HILS_OK
    # every query group is compared: where a near tie (within 1e-3) at the cut lets the selection differ
    # from the oracle's, the set must be one the oracle enumerates for that band and the outputs are
    # compared with the oracle's on that same set
    import parity
    from synth.workloads import Workload
    w = Workload("landmark_feed", B=B, H=H, Hkv=Hkv, N=T, T=T, d=d, C=C, k=k, q_offset=0, dtype="bf16", seed=211)
    arr = {"Q": Q.double().numpy(), "K": K.double().numpy(), "V": V.double().numpy(),
           "L": Ld.double().cpu().numpy()}
    sel_idx = torch.empty((B, Hkv, T, k), dtype=torch.int32, device=DEV)
    sel_score = torch.empty((B, H, T, k + 1), dtype=torch.float32, device=DEV)
    hils.hils_score_select(p, Qd, Ld, sel_idx, sel_score)
    assert hils.hils_sync_status() == hils.HILS_OK
    items = parity.all_items(w)
    sel, sc, o = parity.gather_gpu(w, O, sel_idx, sel_score, items)
    ans = parity.answers_from_arrays(w, arr, items)
    st = parity.compare(w, items, ans, sel, sc, o)
    print({k_: v for k_, v in st.items() if k_ != "fail"})
    assert st["fail"] == [], st["fail"][:5]
