"""The C-ABI library loads and exports every symbol include/hils.h declares; host-side validation (CPU only)."""
import ctypes
import os
import re

import pytest

import chunk_wise_hierarchical_hils_b200 as hils

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "hils.h")).read()
    return sorted(set(re.findall(r"HILS_API\s+[\w\s\*]+?\b(hils_\w+)\s*\(", src)))


def test_header_symbols_exported():
    names = declared_symbols()
    assert len(names) >= 11
    lib = ctypes.CDLL(hils.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(hils.EXPORTS) | set(names)
    assert hils.hils_version() == 122


def test_struct_layout_matches_header():
    # 11 ints + 1 float, no padding
    assert ctypes.sizeof(hils.hils_problem) == 12 * 4


def prob(**kw):
    base = dict(B=2, H=8, Hkv=2, N=256, T=256, d=128, C=64, k=4)
    base.update(kw)
    return hils.problem(**base)


@pytest.mark.parametrize("kw,status", [
    ({}, hils.HILS_OK),
    ({"H": 6, "Hkv": 4}, hils.HILS_ERR_INVALID_ARG),
    ({"N": 0}, hils.HILS_ERR_INVALID_ARG),
    ({"N": 200, "T": 256, "q_offset": 100}, hils.HILS_ERR_INVALID_ARG),
    ({"N": 1, "T": 256, "q_offset": 255}, hils.HILS_OK),
    ({"d": 96}, hils.HILS_ERR_UNSUPPORTED),
    ({"C": 48}, hils.HILS_ERR_UNSUPPORTED),
    ({"k": 65}, hils.HILS_ERR_UNSUPPORTED),
    ({"k": -1}, hils.HILS_ERR_INVALID_ARG),
    ({"H": 64, "Hkv": 2}, hils.HILS_ERR_UNSUPPORTED),
    ({"scale": float("nan")}, hils.HILS_ERR_INVALID_ARG),
    ({"scale": -1.0}, hils.HILS_ERR_INVALID_ARG),
])
def test_validation(kw, status):
    assert hils.hils_validate(prob(**kw)) == status


def test_bad_dtype():
    p = prob()
    p.in_dtype = 7
    assert hils.hils_validate(p) == hils.HILS_ERR_INVALID_ARG


def test_errors_before_launch():
    """Null pointers, misalignment and short workspaces are rejected on the host."""
    p = prob(N=1, T=256, q_offset=255)
    with pytest.raises(hils.HilsError) as e:
        hils.hils_forward(p, 0, 16, 16, 16, 16, (16, 1 << 30), stream=0)
    assert e.value.status == hils.HILS_ERR_INVALID_ARG
    with pytest.raises(hils.HilsError) as e:
        hils.hils_forward(p, 24, 16, 16, 16, 16, (16, 1 << 30), stream=0)
    assert e.value.status == hils.HILS_ERR_INVALID_ARG
    need = hils.hils_forward_workspace_size(p)
    with pytest.raises(hils.HilsError) as e:
        hils.hils_forward(p, 16, 16, 16, 16, 16, (16, need - 1), stream=0)
    assert e.value.status == hils.HILS_ERR_WORKSPACE
    with pytest.raises(hils.HilsError) as e:
        hils.hils_score_select(prob(), 16, 16, 0, 16, stream=0)
    assert e.value.status == hils.HILS_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,args,status", [
    ({"d": 96}, (16, 16, 16, 16, 0, 4), hils.HILS_ERR_UNSUPPORTED),
    ({"C": 0}, (16, 16, 16, 16, 0, 4), hils.HILS_ERR_INVALID_ARG),
    ({}, (16, 16, 16, 16, 0, 5), hils.HILS_ERR_INVALID_ARG),         # c_end past the last chunk (T/C = 4)
    ({}, (16, 16, 16, 16, 3, 2), hils.HILS_ERR_INVALID_ARG),         # c_end < c_begin
    ({}, (16, 16, 16, 16, -1, 2), hils.HILS_ERR_INVALID_ARG),
    ({}, (0, 16, 16, 16, 0, 4), hils.HILS_ERR_INVALID_ARG),          # K null
    ({}, (16, 16, 24, 16, 0, 4), hils.HILS_ERR_INVALID_ARG),         # L misaligned
    ({}, (16, 16, 32, 18, 0, 4), hils.HILS_ERR_INVALID_ARG),         # beta misaligned
    ({"scale": float("inf")}, (16, 16, 16, 16, 0, 4), hils.HILS_ERR_INVALID_ARG),
])
def test_landmarks_errors_before_launch(kw, args, status):
    """hils_landmarks checks its shape, range and pointers on the host; only B, Hkv, T, d, C, dtype, scale count."""
    p = prob(**kw)
    K, U, L, beta, c0, c1 = args
    with pytest.raises(hils.HilsError) as e:
        hils.hils_landmarks(p, K, U, L, beta, c0, c1, stream=0)
    assert e.value.status == status


def test_landmarks_empty_range_launches_nothing():
    # fields the call does not use may hold anything; an empty chunk range returns at once
    p = prob(H=3, N=0, k=-5, C=7)
    hils.hils_landmarks(p, 16, 16, 32, None, 2, 2, stream=0)


@pytest.mark.parametrize("kw,wc,status", [
    ({}, 0, hils.HILS_ERR_INVALID_ARG),                  # a window holds at least the own chunk
    ({"k": 60}, 6, hils.HILS_ERR_UNSUPPORTED),           # k + wc - 1 = 65 past slots
    ({"d": 96}, 2, hils.HILS_ERR_UNSUPPORTED),
    ({"C": 48}, 2, hils.HILS_ERR_UNSUPPORTED),
])
def test_window_validation(kw, wc, status):
    with pytest.raises(hils.HilsError) as e:
        hils.hils_forward_window_workspace_size(prob(**kw), wc)
    assert e.value.status == status
    with pytest.raises(hils.HilsError) as e:
        hils.hils_score_select_window(prob(**kw), wc, None, 16, 16, 16, 16, stream=0)
    assert e.value.status == status


def test_window_errors_before_launch():
    p = prob()
    with pytest.raises(hils.HilsError) as e:       # bias misaligned
        hils.hils_score_select_window(p, 2, 18, 16, 16, 16, 16, stream=0)
    assert e.value.status == hils.HILS_ERR_INVALID_ARG
    with pytest.raises(hils.HilsError) as e:       # sel_idx missing while k + wc - 1 > 0
        hils.hils_score_select_window(p, 2, None, 16, 16, None, 16, stream=0)
    assert e.value.status == hils.HILS_ERR_INVALID_ARG
    need = hils.hils_forward_window_workspace_size(p, 3)
    with pytest.raises(hils.HilsError) as e:
        hils.hils_forward_window(p, 3, None, 16, 16, 16, 16, 16, (16, need - 1), stream=0)
    assert e.value.status == hils.HILS_ERR_WORKSPACE


def test_window_workspace_covers_the_wider_selection():
    # the window adds wc - 1 past slots per query: the workspace holds their indices and scores
    p = prob()
    one, three = hils.hils_forward_window_workspace_size(p, 1), hils.hils_forward_window_workspace_size(p, 3)
    assert one == hils.hils_forward_workspace_size(p)
    assert three >= one + 2 * 2 * 256 * 4 + 2 * 8 * 256 * 4 * 2


@pytest.mark.parametrize("kw", [dict(), dict(N=1, T=131072, q_offset=131071, B=4, H=32, Hkv=8, k=32)])
def test_window_workspace_is_the_attention_of_the_wider_selection(kw):
    # hils_forward_window = window selection (no scratch) + hils_chunk_attend_fuse on k' = k + wc - 1 slots:
    # its workspace holds sel_idx [.., k'] and sel_score [.., k' + 1] (256-byte aligned) and the attention's
    p = prob(**kw)
    wc = 4
    pk = prob(**dict(kw, k=p.k + wc - 1))
    B, H, Hkv, N, kp = p.B, p.H, p.Hkv, p.N, p.k + wc - 1
    up = lambda x: (x + 255) // 256 * 256
    want = up(B * Hkv * N * kp * 4) + up(B * H * N * (kp + 1) * 4) + hils.hils_chunk_attend_fuse_workspace_size(pk)
    assert hils.hils_forward_window_workspace_size(p, wc) == want


def test_workspace_sizes():
    p = prob()
    assert hils.hils_score_select_workspace_size(p) == 0
    assert hils.hils_forward_workspace_size(p) >= 2 * 2 * 256 * 4 * 4 + 2 * 8 * 256 * 5 * 4
    pd = prob(B=16, H=32, Hkv=8, N=1, T=131072, k=32, q_offset=131071)
    assert hils.hils_score_select_workspace_size(pd) > 0
    assert hils.hils_forward_workspace_size(pd) >= max(hils.hils_score_select_workspace_size(pd),
                                                       hils.hils_chunk_attend_fuse_workspace_size(pd))
    with pytest.raises(hils.HilsError):
        hils.hils_forward_workspace_size(prob(d=80))


def test_status_strings():
    for s in range(6):
        assert hils.hils_status_string(s).startswith("HILS_")
    assert "unknown" in hils.hils_status_string(99)


def test_header_is_plain_c_and_links(tmp_path):
    """A C99 program that includes only the header compiles, links against the library and calls it
    (no GPU work: the version and a status string)."""
    import subprocess
    src = tmp_path / "use_hils.c"
    src.write_text(
        '#include "hils.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        "    hils_problem p = {0};\n"
        "    size_t bytes = 0;\n"
        "    (void)p; (void)bytes;\n"
        '    printf("%d %s\\n", hils_version(), hils_status_string(HILS_OK));\n'
        "    return 0;\n"
        "}\n")
    exe = tmp_path / "use_hils"
    libdir = os.path.dirname(hils.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-L", libdir, "-lhils", "-Wl,-rpath," + libdir, "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out[0] == "122"


def _bf16(**kw):
    p = prob(**kw)
    p.in_dtype = hils.HILS_BF16
    p.out_dtype = hils.HILS_BF16
    return p


@pytest.mark.parametrize("kw,env,want", [
    # 8K prefill, k = 16: every landmark tile fits TMEM, the union kernel (visible / selected about 4)
    (dict(B=4, H=32, Hkv=8, N=8192, T=8192, k=16), {}, "select=tc-heads-resident attend=union-tc"),
    (dict(B=4, H=32, Hkv=8, N=8192, T=8192, k=16), {"HILS_SELECT_RESIDENT": "0"}, "select=tc-heads attend=union-tc"),
    (dict(B=4, H=32, Hkv=8, N=8192, T=8192, k=16), {"HILS_PREFILL_ATTEND": "chunk"},
     "select=tc-heads-resident attend=chunk-major"),
    # 256K prefill, k = 32: the per-query selection (k > 16) and chunk-major attention (ratio about 62)
    (dict(B=1, H=16, Hkv=4, N=262144, T=262144, k=32), {}, "select=tc-queries attend=chunk-major"),
    (dict(B=1, H=16, Hkv=4, N=262144, T=262144, k=32), {"HILS_PREFILL_ATTEND": "union"},
     "select=tc-queries attend=union-tc"),
    # single-token decode (the fused kernel needs a device, so forward is not checked here)
    (dict(B=16, H=32, Hkv=8, N=1, T=131072, q_offset=131071, k=32), {}, "select=decode-scan attend=decode-mma"),
])
def test_describe(kw, env, want, monkeypatch):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    text = hils.hils_describe(_bf16(**kw))
    assert text.startswith("forward=")
    assert text.split(" ", 1)[1] == want, text


def test_describe_float32_and_errors():
    p = prob()
    p.in_dtype = hils.HILS_F32
    p.out_dtype = hils.HILS_F32
    assert hils.hils_describe(p).endswith("select=cuda-cores attend=cuda-cores")
    buf = ctypes.create_string_buffer(8)
    lib = ctypes.CDLL(hils.LIB_PATH)
    assert lib.hils_describe(ctypes.byref(prob()), buf, ctypes.c_size_t(8)) == hils.HILS_ERR_INVALID_ARG
    assert lib.hils_describe(ctypes.byref(prob()), None, ctypes.c_size_t(64)) == hils.HILS_ERR_INVALID_ARG
    assert lib.hils_describe(ctypes.byref(prob(N=0)), buf, ctypes.c_size_t(8)) == hils.HILS_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,slices", [
    (dict(B=4, H=32, Hkv=8, N=8192, T=8192, k=16), 8),     # 32 (b, g) units, 4 per slice
    (dict(B=1, H=16, Hkv=4, N=4096, T=4096, k=8), 4),      # one group per slice
    (dict(B=3, H=8, Hkv=2, N=256, T=256, k=4), 6),
    (dict(B=16, H=32, Hkv=8, N=1, T=4096, q_offset=4095, k=8), 8),   # whole batch elements per slice
])
def test_forward_host_workspace(kw, slices):
    """Two device slots of one slice's Q, K, V, L, O plus the slice forward's workspace."""
    p = _bf16(**kw)
    need = hils.hils_forward_host_workspace_size(p)
    b, hkv = kw["B"], kw["Hkv"]
    per = b * hkv // slices
    g = kw["H"] // hkv
    nl = -(-kw["T"] // 64)
    slot = sum(-(-x // 256) * 256 for x in (per * g * kw["N"] * 128 * 2, per * kw["T"] * 128 * 2,
                                            per * kw["T"] * 128 * 2, per * nl * 128 * 2, per * g * kw["N"] * 128 * 2))
    q = _bf16(**dict(kw, B=per // hkv if per >= hkv else 1, Hkv=min(per, hkv), H=min(per, hkv) * g))
    fwd = -(-hils.hils_forward_workspace_size(q) // 256) * 256
    assert need == 2 * slot + fwd


def test_forward_host_errors():
    """Host-side checks before any copy: NULL host pointers, a short workspace, a bad problem."""
    lib = ctypes.CDLL(hils.LIB_PATH)
    p = _bf16()
    need = hils.hils_forward_host_workspace_size(p)
    fake = ctypes.c_void_p(4096)   # never dereferenced: the call returns before any copy
    args = [fake] * 5
    assert lib.hils_forward_host(ctypes.byref(p), None, *args[1:], fake, ctypes.c_size_t(need), None) == \
        hils.HILS_ERR_INVALID_ARG
    assert lib.hils_forward_host(ctypes.byref(p), *args, fake, ctypes.c_size_t(need - 16), None) == \
        hils.HILS_ERR_WORKSPACE
    assert lib.hils_forward_host(ctypes.byref(prob(N=0)), *args, fake, ctypes.c_size_t(need), None) == \
        hils.HILS_ERR_INVALID_ARG
    assert lib.hils_forward_host_workspace_size(ctypes.byref(p), None) == hils.HILS_ERR_INVALID_ARG


def test_every_export_has_argument_types():
    """Each exported entry point taking arguments has ctypes argument types (an untyped pointer argument
    would be passed as a 32-bit int)."""
    src = open(os.path.join(ROOT, "include", "hils.h")).read()
    for n in declared_symbols():
        m = re.search(r"\b" + n + r"\s*\(([^)]*)\)", src)
        if m and m.group(1).strip() not in ("", "void"):
            assert getattr(hils._lib, n).argtypes is not None, n
