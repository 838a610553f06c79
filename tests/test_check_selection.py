"""The debug check of a caller-supplied selection (HILS_CHECK_SELECTION=1) on the GPU.

hils_chunk_attend_fuse trusts sel_idx: every entry -1 or a past chunk of its query, no chunk twice in a
row.  With the check on, a valid selection goes through unchanged (same output bits) and a row that
breaks the rule makes the call return HILS_ERR_INVALID_ARG with nothing else launched.  The planted
entries stay inside the tensors (a chunk at or after the query's own, a repeat), so that even an
unchecked launch would only compute a wrong result.
"""
import pytest
import torch

import chunk_wise_hierarchical_hils_b200 as hils
import parity
from synth import workloads as W
from synth.workloads import Workload

pytestmark = pytest.mark.gpu

W1 = Workload("check_selection", B=1, H=8, Hkv=2, N=640, T=640, d=128, C=64, k=4, q_offset=0, dtype="bf16",
              seed=160, l_mode="chunkmean")


def _setup():
    inp = W.full_inputs(W1)
    dev = {k: parity.to_device(v[1], W1.dtype) for k, v in inp.items()}
    p = parity.problem_of(W1)
    sel_idx = torch.empty((W1.B, W1.Hkv, W1.N, W1.k), dtype=torch.int32, device="cuda")
    sel_score = torch.empty((W1.B, W1.H, W1.N, W1.k + 1), dtype=torch.float32, device="cuda")
    hils.hils_score_select(p, dev["Q"], dev["L"], sel_idx, sel_score,
                           torch.empty(max(hils.hils_score_select_workspace_size(p), 1), dtype=torch.uint8,
                                       device="cuda"))
    ws = torch.empty(max(hils.hils_chunk_attend_fuse_workspace_size(p), 1), dtype=torch.uint8, device="cuda")
    return p, dev, sel_idx, sel_score, ws


def _attend(p, dev, sel_idx, sel_score, ws):
    O = torch.zeros((W1.B, W1.H, W1.N, W1.d), dtype=torch.float32, device="cuda")
    hils.hils_chunk_attend_fuse(p, dev["Q"], dev["K"], dev["V"], sel_idx, sel_score, O, ws)
    assert hils.hils_sync_status() == hils.HILS_OK
    return O


def test_valid_selection_passes_unchanged(monkeypatch):
    p, dev, sel_idx, sel_score, ws = _setup()
    O0 = _attend(p, dev, sel_idx, sel_score, ws)
    monkeypatch.setenv("HILS_CHECK_SELECTION", "1")
    O1 = _attend(p, dev, sel_idx, sel_score, ws)
    assert torch.equal(O0, O1)


@pytest.mark.parametrize("plant", ["own_chunk", "future_chunk", "repeat"])
def test_invalid_selection_is_refused(monkeypatch, plant):
    p, dev, sel_idx, sel_score, ws = _setup()
    i = 300                                    # own chunk 4; chunks 0..3 are its past
    if plant == "own_chunk":
        sel_idx[0, 1, i, 2] = 4
    elif plant == "future_chunk":
        sel_idx[0, 0, i, 0] = 7                # inside the tensors (10 chunks), after the query
    else:
        sel_idx[0, 1, i, 1] = int(sel_idx[0, 1, i, 0])
    monkeypatch.setenv("HILS_CHECK_SELECTION", "1")
    O = torch.zeros((W1.B, W1.H, W1.N, W1.d), dtype=torch.float32, device="cuda")
    with pytest.raises(hils.HilsError) as e:
        hils.hils_chunk_attend_fuse(p, dev["Q"], dev["K"], dev["V"], sel_idx, sel_score, O, ws)
    assert e.value.status == hils.HILS_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(O)) == 0   # nothing was launched
