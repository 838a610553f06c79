"""Bounded waits of the tensor-core kernel: a limit too short for any barrier to
complete makes every CTA give up; the host reads HILS_ERR_TIMEOUT, and the
context stays usable (the next call with the default limit is correct)."""
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
import parity
from synth.workloads import Workload

pytestmark = pytest.mark.gpu


def test_timeout_reported_and_context_usable():
    w = Workload("timeout", B=1, H=8, Hkv=2, N=1024, T=1024, d=128, C=64, k=4, q_offset=0, dtype="bf16",
                 seed=150, l_mode="chunkmean")
    try:
        hils.hils_set_wait_limit(1)          # 1 ns: no barrier phase can complete in time
        O = torch.full((w.B, w.H, w.N, w.d), 5.0, dtype=torch.float32, device="cuda")
        from synth import workloads as W
        inp = W.full_inputs(w)
        dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
        p = parity.problem_of(w)
        ws = torch.empty(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
        hils.hils_forward(p, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws)
        assert hils.hils_sync_status() == hils.HILS_ERR_TIMEOUT
        assert hils.hils_sync_status() == hils.HILS_OK      # the status was cleared by the read
    finally:
        hils.hils_set_wait_limit(0)
    st, _ = parity.run_small(w)
    assert st["fail"] == [], st["fail"][:3]
