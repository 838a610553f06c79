"""hils_forward_host (host buffers in and out, slices of (batch, kv-group) pairs with copies and compute
overlapped) returns what hils_forward returns on the same inputs held on the device, and what the oracle
computes.

The (batch, kv-group) pairs are independent problems ("Hierarchical Sparse Attention Done Right", Sec. 4
"Architecture": a group's heads share one selection, groups share nothing), so a slice's forward is the
whole-batch forward restricted to its pairs: bit for bit on the kernels whose arithmetic does not depend
on the batch (the union and CUDA-core attentions, every selection), within float32 rounding on the
chunk-major attention (its partial outputs add in no fixed order) and on single-token decode (the CTAs
per pair depend on the pairs per call).
"""
import numpy as np
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
import parity
from synth import workloads as W
from synth.workloads import Workload

pytestmark = pytest.mark.gpu


def wl(name, **kw):
    base = dict(B=2, H=8, Hkv=2, N=512, T=512, d=128, C=64, k=4, q_offset=0, dtype="bf16", seed=160,
                l_mode="chunkmean")
    base.update(kw)
    return Workload(name, **base)


CASES = [
    (wl("union_b3_g4", B=3, H=8, Hkv=2, N=700, T=700, k=5), None),
    (wl("chunked_prefill", B=2, H=16, Hkv=4, N=256, T=1024, q_offset=768, k=6, seed=161), None),
    (wl("chunk_major_forced", B=2, H=8, Hkv=2, N=1000, T=1000, k=3, seed=162), "chunk"),
    (wl("f32_cuda_cores", B=2, H=4, Hkv=2, N=300, T=300, k=2, dtype="f32", seed=163), None),
    (wl("decode_b5", B=5, H=8, Hkv=2, N=1, T=3000, q_offset=2999, k=8, seed=164), None),
    (wl("one_unit", B=1, H=4, Hkv=1, N=400, T=400, k=4, seed=165), None),
]


@pytest.mark.parametrize("w,attend", CASES, ids=lambda c: c.name if isinstance(c, Workload) else str(c))
def test_forward_host_equals_device_forward(w, attend, monkeypatch):
    if attend:
        monkeypatch.setenv("HILS_PREFILL_ATTEND", attend)
    inp = W.full_inputs(w)
    dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
    O_dev, _, _ = parity.gpu_run(w, dev)
    p = parity.problem_of(w)
    host = {k: v.cpu().pin_memory() for k, v in dev.items()}
    O_host = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.float32).pin_memory()
    ws = torch.empty(hils.hils_forward_host_workspace_size(p), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    hils.hils_forward_host(p, host["Q"], host["K"], host["V"], host["L"], O_host, ws, stream)
    stream.synchronize()
    assert hils.hils_sync_status() == hils.HILS_OK
    got, want = O_host.numpy(), O_dev.cpu().numpy()
    assert np.isfinite(got).all()
    if attend == "chunk" or w.N == 1:
        # chunk-major partial outputs add in no fixed order; single-token decode splits a (b, g) over a
        # number of CTAs that depends on how many pairs the call holds, and adds their partials in order
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)
    else:
        assert np.array_equal(got, want)
    # and against the oracle, every query group
    items = parity.all_items(w)
    sel_idx = torch.empty((w.B, w.Hkv, w.N, max(w.k, 1)), dtype=torch.int32, device="cuda")
    sel_score = torch.empty((w.B, w.H, w.N, w.k + 1), dtype=torch.float32, device="cuda")
    ws_sel = torch.empty(max(hils.hils_score_select_workspace_size(p), 1), dtype=torch.uint8, device="cuda")
    hils.hils_score_select(p, dev["Q"], dev["L"], sel_idx, sel_score, ws_sel)
    sel, s, o = parity.gather_gpu(w, O_host.cuda(), sel_idx, sel_score, items)
    ans = parity.answers_from_arrays(w, {k: v[0] for k, v in inp.items()}, items)
    st = parity.compare(w, items, ans, sel, s, o)
    assert st["fail"] == [], st["fail"][:5]


def test_forward_host_repeated_calls_reuse_slots():
    """Back-to-back calls on one stream (the internal events are re-recorded call after call) and a
    second problem size in between: every call's output is the device forward's."""
    w1 = wl("repeat_a", B=4, H=8, Hkv=2, N=512, T=512, k=4, seed=166)
    w2 = wl("repeat_b", B=1, H=8, Hkv=2, N=256, T=256, k=2, seed=167)
    outs = []
    for w in (w1, w2, w1):
        inp = W.full_inputs(w)
        dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
        O_dev, _, _ = parity.gpu_run(w, dev)
        p = parity.problem_of(w)
        host = {k: v.cpu().pin_memory() for k, v in dev.items()}
        O_host = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32).pin_memory()
        ws = torch.empty(hils.hils_forward_host_workspace_size(p), dtype=torch.uint8, device="cuda")
        for _ in range(3):
            hils.hils_forward_host(p, host["Q"], host["K"], host["V"], host["L"], O_host, ws)
        torch.cuda.synchronize()
        outs.append(np.array_equal(O_host.numpy(), O_dev.cpu().numpy()))
    assert outs == [True, True, True]
