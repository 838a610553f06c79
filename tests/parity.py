"""GPU-vs-oracle comparison helpers shared by the GPU parity tests.

The GPU selection must equal the oracle's, except where the oracle itself finds
a near tie (two candidate group scores within EPS_TIE of the k-th kept score):
then any of the selections the oracle enumerates for that band is accepted, and
the outputs are compared with the oracle's outputs for that same selection.
The oracle never receives anything computed on the GPU.
"""
import numpy as np
import torch

import chunk_wise_hierarchical_hils_b200 as hils
from oracle import oracle as orc
from synth import workloads as W

EPS_TIE = 1e-3          # near-tie band on group scores (selection may differ inside it)
TOL_O = {"f32": 1e-4, "bf16": 1e-2}   # max-abs output error of the float32 result
# A bf16 output adds its own rounding, up to half a bf16 ulp of the value (2^-8 relative below the
# next power of two): compared against the float64 result, a bf16 output may differ by the
# computation's tolerance plus that half ulp.  (For |o| >= 4 the half ulp alone is >= 0.0078, so a
# flat 1e-2 cannot hold for bf16 outputs even from an exact computation.)
TOL_S = 1e-4            # max-abs error of the per-head slot scores


def to_device(raw, dtype):
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(raw)).cuda()
    return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()


def problem_of(w, out_dtype="f32"):
    dt = {"f32": hils.HILS_F32, "bf16": hils.HILS_BF16}
    return hils.problem(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.k, w.q_offset, dt[w.dtype], dt[out_dtype])


def gpu_run(w, dev, out_dtype="f32", stepwise=False):
    """Run the library on device inputs dev = {Q, K, V, L}; returns (O, sel_idx, sel_score) on the device."""
    p = problem_of(w, out_dtype)
    odt = torch.float32 if out_dtype == "f32" else torch.bfloat16
    O = torch.empty((w.B, w.H, w.N, w.d), dtype=odt, device="cuda")
    sel_idx = torch.empty((w.B, w.Hkv, w.N, max(w.k, 1)), dtype=torch.int32, device="cuda")
    sel_score = torch.empty((w.B, w.H, w.N, w.k + 1), dtype=torch.float32, device="cuda")
    ws_sel = torch.empty(max(hils.hils_score_select_workspace_size(p), 1), dtype=torch.uint8, device="cuda")
    hils.hils_score_select(p, dev["Q"], dev["L"], sel_idx, sel_score, ws_sel)
    if stepwise:
        ws_att = torch.empty(max(hils.hils_chunk_attend_fuse_workspace_size(p), 1), dtype=torch.uint8, device="cuda")
        hils.hils_chunk_attend_fuse(p, dev["Q"], dev["K"], dev["V"], sel_idx, sel_score, O, ws_att)
    else:
        ws = torch.empty(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
        hils.hils_forward(p, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws)
    assert hils.hils_sync_status() == hils.HILS_OK
    return O, sel_idx[..., :w.k], sel_score


def answers_from_arrays(w, arr, items, eps=EPS_TIE):
    """Oracle answers for items [(b, g, i)] from whole float64 arrays arr = {Q, K, V, L}."""
    scale = orc.default_scale(w.d)
    out = []
    for (b, g, i) in items:
        q = arr["Q"][b, g * w.G:(g + 1) * w.G, i, :]

        def fetch(c, b=b, g=g):
            t0, t1 = c * w.C, min((c + 1) * w.C, w.T)
            return arr["K"][b, g, t0:t1], arr["V"][b, g, t0:t1]

        out.append(orc.evaluate_query(q, arr["L"][b, g], fetch, w.C, w.k, w.q_offset + i, scale, eps))
    return out


def gather_gpu(w, O, sel_idx, sel_score, items):
    """Copy the rows of the sampled query groups to the host (float64 / int)."""
    b = torch.tensor([it[0] for it in items], device="cuda")
    g = torch.tensor([it[1] for it in items], device="cuda")
    i = torch.tensor([it[2] for it in items], device="cuda")
    heads = g[:, None] * w.G + torch.arange(w.G, device="cuda")[None, :]
    o = O[b[:, None], heads, i[:, None]].double().cpu().numpy()              # [n, G, d]
    s = sel_score[b[:, None], heads, i[:, None]].double().cpu().numpy()      # [n, G, k+1]
    sel = sel_idx[b, g, i].cpu().numpy() if w.k > 0 else np.zeros((len(items), 0), np.int32)
    return sel, s, o


def compare(w, items, answers, sel, s, o, tol_o=None, tol_s=TOL_S, out_dtype="f32"):
    """Check every sampled query group; returns a stats dict (failures listed in stats['fail']).

    tol_o: the output bound, one number for every item or a sequence with one per item."""
    if tol_o is None:
        tol_o = TOL_O[w.dtype]
    tol_items = list(tol_o) if np.ndim(tol_o) else [tol_o] * len(items)
    st = {"n": len(items), "near_tie": 0, "overflow": 0, "max_err_O": 0.0, "max_err_s": 0.0, "fail": []}
    for n, (it, ans) in enumerate(zip(items, answers)):
        pos = ans["pos"]
        ci = pos // w.C
        gsel = [int(c) for c in sel[n]]
        gset = set(c for c in gsel if c >= 0)
        m = min(w.k, ci)
        if len(gset) != m or sum(1 for c in gsel if c < 0) != w.k - m or sorted(gsel[:m]) != sorted(gset):
            st["fail"].append((it, "bad padding / duplicates", gsel))
            continue
        if any(c < 0 or c >= ci for c in gset):
            st["fail"].append((it, "chunk outside the past range", gsel))
            continue
        match = None
        for a, alt in enumerate(ans["alts"]):
            if set(int(c) for c in alt[0][:w.k] if c >= 0) == gset:
                match = a
                break
        if match is None:
            prim = [int(c) for c in ans["alts"][0][0][:w.k]]
            diff = sorted(gset ^ set(c for c in prim if c >= 0))
            st["fail"].append((it, "selection differs", gsel, prim, [(c, ans["shat"][c]) for c in diff]))
            continue
        if match > 0:
            st["near_tie"] += 1
        st["overflow"] += int(ans["overflow"])
        # rank order: descending group score, ties and near ties within EPS_TIE allowed
        sh = ans["shat"]
        for j in range(m - 1):
            if sh[gsel[j]] < sh[gsel[j + 1]] - EPS_TIE:
                st["fail"].append((it, "rank order", gsel))
                break
        full, os_, _, oo = ans["alts"][match]
        # slot scores by chunk index (own chunk = slot k)
        idx = {int(c): j for j, c in enumerate(full[:w.k]) if c >= 0}
        for j, c in enumerate(gsel + [ci]):
            jo = w.k if j == w.k else (idx[c] if c >= 0 else None)
            for h in range(w.G):
                gs = s[n, h, j]
                if jo is None:
                    if gs != -np.inf:
                        st["fail"].append((it, "empty slot score", j, gs))
                    continue
                e = abs(gs - os_[h, jo])
                st["max_err_s"] = max(st["max_err_s"], e)
                if not e <= tol_s:
                    st["fail"].append((it, "slot score", j, h, gs, os_[h, jo]))
        tol_n = tol_items[n]
        allowed = tol_n
        if out_dtype == "bf16":
            allowed = tol_n + np.ldexp(1.0, np.frexp(np.abs(oo))[1] - 9)   # half ulp of bf16 at |o|
        e = np.abs(o[n] - oo)
        st["max_err_O"] = max(st["max_err_O"], float(np.max(e)))
        if not np.all(e <= allowed):
            st["fail"].append((it, "output err %.3g (bound %.3g)" % (float(np.max(e - allowed + tol_n)), tol_n)))
    return st


def all_items(w):
    return [(b, g, i) for b in range(w.B) for g in range(w.Hkv) for i in range(w.N)]


def run_small(w, out_dtype="f32", stepwise=False):
    """Whole-tensor parity on a small workload: every query group is checked."""
    inp = W.full_inputs(w)
    arr = {k: v[0] for k, v in inp.items()}
    dev = {k: to_device(v[1], w.dtype) for k, v in inp.items()}
    O, sel_idx, sel_score = gpu_run(w, dev, out_dtype, stepwise)
    items = all_items(w)
    sel, s, o = gather_gpu(w, O, sel_idx, sel_score, items)
    ans = answers_from_arrays(w, arr, items)
    return compare(w, items, ans, sel, s, o, out_dtype=out_dtype), (O, sel_idx, sel_score)
