"""Bounded waits of the tensor-core kernels: a wait on a barrier nothing signals
(the library's stall-injection test control) expires after the wait limit; the
host reads HILS_ERR_TIMEOUT, and the context stays usable (the next call is
correct).  No GPU fault is involved."""
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
import parity
from synth.workloads import Workload

pytestmark = pytest.mark.gpu


def test_timeout_reported_and_context_usable():
    w = Workload("timeout", B=1, H=8, Hkv=2, N=1024, T=1024, d=128, C=64, k=4, q_offset=0, dtype="bf16",
                 seed=150, l_mode="chunkmean")
    from synth import workloads as W
    inp = W.full_inputs(w)
    dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
    p = parity.problem_of(w)
    O = torch.full((w.B, w.H, w.N, w.d), 5.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    try:
        hils.hils_set_wait_limit(2_000_000)      # 2 ms
        hils.hils_debug_inject_stall(1)
        hils.hils_forward(p, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws)
        assert hils.hils_sync_status() == hils.HILS_ERR_TIMEOUT
        assert hils.hils_sync_status() == hils.HILS_OK      # the status was cleared by the read
    finally:
        hils.hils_debug_inject_stall(0)
        hils.hils_set_wait_limit(0)
    st, _ = parity.run_small(w)
    assert st["fail"] == [], st["fail"][:3]
