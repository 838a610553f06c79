"""The allocation-free decode selection entry point against the regular one.

hils_decode_score_select_noalloc serves callers that cannot allocate device
memory (plugins whose host application owns the whole device memory budget,
memory-capped processes, latency-critical paths that must not enter the
driver's allocator): it takes its scratch from a fixed array inside the
library instead of a caller workspace.  This file is collected last so that a
run stopping at the first failure has already run every other test; it also
passes on its own in a fresh process, where its first call performs the
per-device set-up.
"""
import ctypes

import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
from synth import gpu as synth_gpu
from synth.workloads import Workload

pytestmark = pytest.mark.gpu

TOL_S = 1e-4   # slot-score tolerance used by the parity tests; selections must match exactly


def _wl(name, **kw):
    base = dict(B=4, H=32, Hkv=8, N=1, T=131072, d=128, C=64, k=32, q_offset=131071, dtype="bf16", seed=40,
                l_mode="chunkmean")
    base.update(kw)
    return Workload(name, **base)


CASES = [
    _wl("decode_128k_b4"),
    _wl("decode_1m_needles", B=1, T=1 << 20, q_offset=(1 << 20) - 1, k=64, seed=41, l_mode="iid",
        n_needles=16, needle_period=512),
    _wl("decode_f32_d64_ragged", B=3, H=8, Hkv=2, T=50000, q_offset=49999, d=64, C=32, k=8, dtype="f32", seed=42,
        l_mode="iid"),
]


def _outputs(w):
    sel = torch.full((w.B, w.Hkv, 1, w.k), -7, dtype=torch.int32, device="cuda")
    score = torch.full((w.B, w.H, 1, w.k + 1), 7.0, dtype=torch.float32, device="cuda")
    return sel, score


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_version(w):
    dev = synth_gpu.alloc_inputs(w)
    dt = hils.HILS_BF16 if w.dtype == "bf16" else hils.HILS_F32
    p = hils.problem(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.k, w.q_offset, dt, hils.HILS_F32)
    assert hils.hils_score_select_workspace_size(p) <= hils.HILS_NOALLOC_SCRATCH_BYTES
    ref_sel, ref_score = _outputs(w)
    ws = torch.empty(hils.hils_score_select_workspace_size(p), dtype=torch.uint8, device="cuda")
    hils.hils_score_select(p, dev["Q"], dev["L"], ref_sel, ref_score, ws)
    torch.cuda.synchronize()
    for call in range(2):      # two calls in a row: the shared scratch keeps the previous call's contents
        sel, score = _outputs(w)
        hils.hils_decode_score_select_noalloc(p, dev["Q"], dev["L"], sel, score)
        torch.cuda.synchronize()
        assert torch.equal(sel, ref_sel), "call %d: selection differs" % call
        finite = torch.isfinite(ref_score)
        assert torch.equal(finite, torch.isfinite(score))
        err = (score[finite] - ref_score[finite]).abs().max().item() if finite.any() else 0.0
        assert err <= TOL_S, "call %d: slot score error %g" % (call, err)


def test_noalloc_through_raw_c_abi():
    """Direct ctypes call of the exported symbol, as a C caller would make it."""
    w = CASES[0]
    dev = synth_gpu.alloc_inputs(w)
    lib = ctypes.CDLL(hils.LIB_PATH)
    fn = lib.hils_decode_score_select_noalloc
    fn.argtypes = [ctypes.POINTER(hils.hils_problem)] + [ctypes.c_void_p] * 5
    fn.restype = ctypes.c_int
    p = hils.problem(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.k, w.q_offset, hils.HILS_BF16, hils.HILS_F32)
    ref_sel, ref_score = _outputs(w)
    ws = torch.empty(hils.hils_score_select_workspace_size(p), dtype=torch.uint8, device="cuda")
    hils.hils_score_select(p, dev["Q"], dev["L"], ref_sel, ref_score, ws)
    sel, score = _outputs(w)
    stream = torch.cuda.current_stream().cuda_stream
    assert fn(ctypes.byref(p), dev["Q"].data_ptr(), dev["L"].data_ptr(), sel.data_ptr(), score.data_ptr(),
              stream) == hils.HILS_OK
    torch.cuda.synchronize()
    assert torch.equal(sel, ref_sel)
    assert torch.allclose(score, ref_score, atol=TOL_S, rtol=0)


def test_noalloc_rejects_oversized_and_prefill():
    big = hils.problem(64, 32, 8, 1, 1 << 22, 128, 64, 64, (1 << 22) - 1, hils.HILS_BF16, hils.HILS_F32)
    assert hils.hils_score_select_workspace_size(big) > hils.HILS_NOALLOC_SCRATCH_BYTES
    with pytest.raises(hils.HilsError) as e:
        hils.hils_decode_score_select_noalloc(big, 16, 16, 16, 16)
    assert e.value.status == hils.HILS_ERR_WORKSPACE
    pre = hils.problem(1, 4, 2, 256, 256, 128, 64, 4, 0, hils.HILS_BF16, hils.HILS_F32)
    with pytest.raises(hils.HilsError) as e:
        hils.hils_decode_score_select_noalloc(pre, 16, 16, 16, 16)
    assert e.value.status == hils.HILS_ERR_UNSUPPORTED
