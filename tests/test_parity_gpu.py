"""GPU vs oracle, whole tensors, small shapes that span several tiles and a ragged tail.

Every query group of every case is compared: exact chunk sets (near ties
within 1e-3 excepted, as enumerated by the oracle), slot scores within 1e-4,
outputs within 1e-4 (float32 inputs) or 1e-2 (bf16 inputs).
"""
import numpy as np
import pytest
import torch

import parity
from synth.workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu


def wl(name, **kw):
    base = dict(B=1, H=4, Hkv=2, N=512, T=512, d=128, C=64, k=4, q_offset=0, dtype="bf16", seed=100,
                l_mode="chunkmean")
    base.update(kw)
    return Workload(name, **base)


CASES = [
    WORKLOADS["tiny_f32"],
    wl("g4_d128_c64_ragged", B=2, H=8, Hkv=2, N=1000, T=1000, k=5, seed=101),
    wl("g1_d64_c32", H=2, Hkv=2, N=700, T=700, d=64, C=32, k=7, seed=102, l_mode="iid"),
    wl("g8_d128_c128", H=16, Hkv=2, N=640, T=640, C=128, k=3, seed=103),
    wl("f32_g2_d128_c64", H=4, Hkv=2, N=300, T=300, k=2, dtype="f32", seed=104),
    wl("k0_own_chunk_only", N=333, T=333, k=0, seed=105),
    wl("k16_more_than_visible", N=200, T=200, C=32, k=16, seed=106),
    wl("chunked_prefill_offset", N=256, T=1024, q_offset=768, k=6, seed=107),
    wl("g16", H=16, Hkv=1, N=200, T=200, k=3, seed=108),
    wl("k64_max", H=2, Hkv=1, N=300, T=4200, q_offset=3900, C=32, k=64, seed=109, l_mode="iid"),
    wl("needles", B=1, H=8, Hkv=2, N=2048, T=2048, k=4, seed=110, l_mode="iid", n_needles=8, needle_period=128),
    wl("g1_d128_long", B=1, H=2, Hkv=2, N=1200, T=9000, q_offset=7800, k=12, seed=111),
    wl("g2_k32_c128", B=2, H=4, Hkv=2, N=700, T=4400, q_offset=3700, C=128, k=32, seed=112, l_mode="iid"),
]
DECODE = [
    wl("decode_ragged_T", B=3, H=8, Hkv=2, N=1, T=1000, q_offset=999, k=4, seed=120),
    wl("decode_f32_d64", B=2, H=4, Hkv=1, N=1, T=4096 + 17, q_offset=4096 + 16, d=64, C=32, k=8, dtype="f32",
       seed=121),
    wl("decode_first_chunk", B=2, H=4, Hkv=2, N=1, T=5, q_offset=4, k=4, seed=122),
    wl("decode_k0", B=2, H=4, Hkv=2, N=1, T=700, q_offset=699, k=0, seed=123),
    wl("decode_long_split", B=2, H=8, Hkv=2, N=1, T=64 * 3000 + 5, q_offset=64 * 3000 + 4, k=32, seed=124,
       l_mode="iid"),
    wl("decode_k64_c128", B=1, H=16, Hkv=4, N=1, T=128 * 700, q_offset=128 * 700 - 1, C=128, k=64, seed=125,
       l_mode="iid"),
    wl("decode_g16_partial_chunk", B=2, H=16, Hkv=1, N=1, T=3000, q_offset=2999, k=8, seed=126),
    wl("decode_g1_c128", B=3, H=4, Hkv=4, N=1, T=128 * 40 + 77, q_offset=128 * 40 + 76, C=128, k=5, seed=127),
]


def _check(st):
    assert st["fail"] == [], st["fail"][:5]


@pytest.mark.parametrize("w", CASES + DECODE, ids=lambda w: w.name)
def test_parity_small(w):
    st, _ = parity.run_small(w)
    print(w.name, {k: v for k, v in st.items() if k != "fail"})
    _check(st)


@pytest.mark.parametrize("w", [CASES[1], CASES[7], CASES[8], CASES[10], CASES[11]], ids=lambda w: w.name)
def test_cuda_core_kernel_too(w, monkeypatch):
    """The CUDA-core prefill kernel, forced, on shapes the tensor-core kernel normally takes."""
    monkeypatch.setenv("HILS_PREFILL_KERNEL", "simt")
    st, _ = parity.run_small(w)
    _check(st)


@pytest.mark.parametrize("w", [CASES[1], CASES[3], CASES[5], CASES[6], CASES[7], CASES[8], CASES[9], CASES[10],
                               CASES[11], CASES[12]], ids=lambda w: w.name)
def test_chunk_major_attention_too(w, monkeypatch):
    """The chunk-major tensor-core prefill attention (selection inverted per chunk, gathered query rows,
    partial outputs added in L2), forced, on shapes the union kernel normally takes."""
    monkeypatch.setenv("HILS_PREFILL_ATTEND", "chunk")
    st, _ = parity.run_small(w)
    _check(st)


@pytest.mark.parametrize("w", [CASES[1], CASES[3], CASES[5], CASES[6], CASES[7], CASES[8], CASES[10], CASES[11],
                               CASES[12]], ids=lambda w: w.name)
def test_persistent_union_attention(w, monkeypatch):
    """The union attention as a persistent kernel (one CTA per SM walking query tiles, the next tile's
    chunk union built while the current tile's last products run), forced on the tensor-core cases."""
    monkeypatch.setenv("HILS_PREFILL_KERNEL", "persistent")
    st, _ = parity.run_small(w)
    _check(st)


@pytest.mark.parametrize("attend", ["union", "chunk"])
def test_both_prefill_attentions_with_bf16_output(attend, monkeypatch):
    monkeypatch.setenv("HILS_PREFILL_ATTEND", attend)
    st, _ = parity.run_small(CASES[1], out_dtype="bf16")
    _check(st)


# chunked prefill over 3 and 6 landmark tiles of 64 (256 and 512 resident TMEM columns)
RESIDENT = [
    wl("g4_c32_three_tiles", B=1, H=8, Hkv=2, N=300, T=6000, q_offset=5700, C=32, k=8, seed=113),
    wl("g2_c32_six_tiles", B=1, H=4, Hkv=2, N=260, T=12000, q_offset=11740, C=32, k=16, seed=114, l_mode="iid"),
]


@pytest.mark.parametrize("kernel", ["heads", "heads_streaming", "queries"])
@pytest.mark.parametrize("w", [CASES[1], CASES[3], CASES[5], CASES[6], CASES[7], CASES[8], CASES[10], CASES[11],
                               CASES[12]] + RESIDENT, ids=lambda w: w.name)
def test_both_tensor_core_selections(w, kernel, monkeypatch):
    """Each tensor-core prefill selection forced on shapes the other one may take: one product row per
    head (group score by a butterfly over the heads; with k <= 16 and at most 8 landmark tiles the tiles
    stay in TMEM and the G lanes of a query split the columns, "heads_streaming" forces the per-row
    lists instead) or one per query (group score from the mean query, per-head slot scores after the
    scan)."""
    monkeypatch.setenv("HILS_SELECT_KERNEL", "heads" if kernel.startswith("heads") else kernel)
    if kernel == "heads_streaming":
        monkeypatch.setenv("HILS_SELECT_RESIDENT", "0")
    st, _ = parity.run_small(w)
    _check(st)


@pytest.mark.parametrize("w", [DECODE[0], DECODE[2], DECODE[3], DECODE[4], DECODE[6]], ids=lambda w: w.name)
def test_two_kernel_decode_too(w, monkeypatch):
    """hils_forward's single-token decode on the two kernels (selection, then attention), forced, on shapes
    the fused cooperative kernel normally takes."""
    monkeypatch.setenv("HILS_DECODE_FUSED", "0")
    st, _ = parity.run_small(w)
    _check(st)


@pytest.mark.parametrize("w", [DECODE[0], DECODE[4], DECODE[6]], ids=lambda w: w.name)
def test_fused_decode_selection_equals_the_selection_call(w):
    """The fused decode kernel writes its selection into hils_forward's workspace: it must equal
    hils_score_select's bit for bit (same scores, same order), and its slot scores agree within 1e-6."""
    import chunk_wise_hierarchical_hils_b200 as hils
    from synth import workloads as W
    inp = W.full_inputs(w)
    dev = {k: parity.to_device(v[1], w.dtype) for k, v in inp.items()}
    p = parity.problem_of(w)
    sel_idx = torch.empty((w.B, w.Hkv, 1, w.k), dtype=torch.int32, device="cuda")
    sel_score = torch.empty((w.B, w.H, 1, w.k + 1), dtype=torch.float32, device="cuda")
    ws_sel = torch.empty(max(hils.hils_score_select_workspace_size(p), 1), dtype=torch.uint8, device="cuda")
    hils.hils_score_select(p, dev["Q"], dev["L"], sel_idx, sel_score, ws_sel)
    O = torch.empty((w.B, w.H, 1, w.d), dtype=torch.float32, device="cuda")
    ws = torch.zeros(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    hils.hils_forward(p, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws)
    assert hils.hils_sync_status() == hils.HILS_OK
    # hils_forward keeps the selection at the start of its workspace: sel_idx rows, then (256-byte
    # aligned) the slot scores
    n_idx = w.B * w.Hkv * w.k
    off = (n_idx * 4 + 255) // 256 * 256
    f_idx = ws[:n_idx * 4].view(torch.int32).view(w.B, w.Hkv, 1, w.k)
    f_score = ws[off:off + w.B * w.H * (w.k + 1) * 4].view(torch.float32).view(w.B, w.H, 1, w.k + 1)
    assert torch.equal(f_idx, sel_idx)
    fin = torch.isfinite(sel_score)
    assert torch.equal(fin, torch.isfinite(f_score))
    assert float((f_score[fin] - sel_score[fin]).abs().max()) <= 1e-6


@pytest.mark.parametrize("w", [DECODE[0], DECODE[2], DECODE[4], DECODE[5]], ids=lambda w: w.name)
def test_cuda_core_decode_too(w, monkeypatch):
    """The CUDA-core decode attention kernel, forced, on shapes the tensor-core tile kernel normally takes."""
    monkeypatch.setenv("HILS_DECODE_KERNEL", "simt")
    st, _ = parity.run_small(w)
    _check(st)


@pytest.mark.parametrize("w", [CASES[1], DECODE[0], DECODE[5]], ids=lambda w: w.name)
def test_bf16_output(w):
    st, _ = parity.run_small(w, out_dtype="bf16")
    _check(st)


@pytest.mark.parametrize("w", [CASES[1], CASES[4], DECODE[1]], ids=lambda w: w.name)
def test_stepwise_equals_forward(w):
    st, (O1, s1, c1) = parity.run_small(w, stepwise=True)
    _check(st)
    _, (O2, s2, c2) = parity.run_small(w, stepwise=False)
    assert torch.equal(O1, O2) and torch.equal(s1, s2) and torch.equal(c1, c2)


def test_exact_ties_lowest_index():
    """Planted exact duplicate landmarks: ties go to the lower chunk index, bit-exactly."""
    w = wl("ties", B=1, H=4, Hkv=1, N=1024, T=1024, C=32, k=6, seed=130, l_mode="iid")
    from synth import workloads as W
    inp = W.full_inputs(w)
    arr = {k: v[0].copy() for k, v in inp.items()}
    raw = {k: v[1].copy() for k, v in inp.items()}
    # landmark of chunk c = level[c % 5] * (mean query direction): five well separated score levels
    qbar = arr["Q"][0].mean(axis=(0, 1))
    levels = np.array([0.5, -1.0, 2.0, 0.0, 1.0])
    from synth.philox import f64_to_f32, f32_to_bf16_bits, bf16_bits_to_f64
    for c in range(w.nL):
        bits = f32_to_bf16_bits(f64_to_f32(levels[c % 5] * qbar * 4.0))
        raw["L"][0, 0, c] = bits
        arr["L"][0, 0, c] = bf16_bits_to_f64(bits)
    dev = {k: parity.to_device(v, w.dtype) for k, v in raw.items()}
    O, sel_idx, sel_score = parity.gpu_run(w, dev)
    items = parity.all_items(w)
    sel, s, o = parity.gather_gpu(w, O, sel_idx, sel_score, items)
    ans = parity.answers_from_arrays(w, arr, items, eps=0.0)
    for n, a in enumerate(ans):
        prim = [int(c) for c in a["alts"][0][0][:w.k]]
        assert [int(c) for c in sel[n]] == prim, (items[n], sel[n], prim)
    st = parity.compare(w, items, ans, sel, s, o)
    _check(st)


@pytest.mark.parametrize("attend", ["union", "chunk", "persistent"])
def test_large_and_tiny_values(attend, monkeypatch):
    """V entries far outside N(0,1): +-1e5 (beyond f16's range), +-3e4 (inside it) and +-1e-6 (f16
    subnormals), planted in a few chunks of some (b, kv-head) slices, so that most rows of the blocks
    that load those chunks did not select them.  The output is defined for every finite input
    ("Hierarchical Sparse Attention Done Right", Sec. 3, "Hierarchical softmax"): no row may be
    poisoned, and every row must match the oracle.

    Bound per row: the value product rounds P to 16 bits (f16, relative 2^-11, or bf16, 2^-9, for a
    slice holding a value beyond f16's range) and V enters it exactly, so the error from that rounding
    is at most 2^-9 times the largest |v| the row attends to (its P sums to one).  Rows that attend to
    |v| <= 8 only keep the usual 1e-2; rows that attend to a planted large value get 2^-8 times it."""
    from synth import workloads as W
    from synth.philox import f64_to_f32, f32_to_bf16_bits, bf16_bits_to_f64
    if attend == "persistent":
        monkeypatch.setenv("HILS_PREFILL_KERNEL", "persistent")
    else:
        monkeypatch.setenv("HILS_PREFILL_ATTEND", attend)
    w = wl("wide_values", B=2, H=8, Hkv=2, N=1024, T=1024, k=4, seed=140)
    inp = W.full_inputs(w)
    arr = {k: v[0].copy() for k, v in inp.items()}
    raw = {k: v[1].copy() for k, v in inp.items()}

    def plant(b, g, c, rows, cols, values):
        for r_, c_, v_ in zip(rows, cols, values):
            t = c * w.C + r_
            bits = f32_to_bf16_bits(f64_to_f32(np.array([v_], dtype=np.float64)))[0]
            raw["V"][b, g, t, c_] = bits
            arr["V"][b, g, t, c_] = bf16_bits_to_f64(np.array([bits]))[0]

    rng = np.random.default_rng(141)

    def some(n, mag):
        return (rng.integers(0, w.C, n), rng.integers(0, w.d, n), mag * rng.choice([-1.0, 1.0], n))

    plant(0, 0, 5, *some(6, 1e5))          # slice (0, 0): beyond f16 -> the bf16 value product
    plant(0, 1, 9, *some(6, 3e4))          # slice (0, 1): large but exact in f16
    plant(1, 0, 3, *some(200, 1e-6))       # slice (1, 0): f16 subnormals
    plant(1, 1, 12, *some(4, 1e5))         # slice (1, 1): both
    plant(1, 1, 14, *some(200, 1e-6))
    dev = {k: parity.to_device(v, w.dtype) for k, v in raw.items()}
    O, sel_idx, sel_score = parity.gpu_run(w, dev)
    assert torch.isfinite(O).all()
    items = parity.all_items(w)
    sel, s, o = parity.gather_gpu(w, O, sel_idx, sel_score, items)
    ans = parity.answers_from_arrays(w, arr, items)
    tol = []
    for n, (b, g, i) in enumerate(items):
        chunks = [int(c) for c in sel[n] if c >= 0] + [(w.q_offset + i) // w.C]
        vmax = max(float(np.max(np.abs(arr["V"][b, g, c * w.C:(c + 1) * w.C]))) for c in chunks)
        tol.append(parity.TOL_O["bf16"] if vmax <= 8.0 else 2.0 ** -8 * vmax)
    st = parity.compare(w, items, ans, sel, s, o, tol_o=tol)
    print({k: v for k, v in st.items() if k != "fail"}, "rows with a planted value:", sum(t > 0.01 for t in tol))
    assert sum(t > 0.01 for t in tol) > 20     # the planted chunks were attended by some rows
    _check(st)
