"""Host-side pieces of the benchmark (CPU): the algorithmic work and bytes it reports, and the rule
that an ncu traffic figure is used only for the kernel sources it was captured on."""
import hashlib
import importlib.util
import json
import os

import pytest

from synth.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_figures_of_the_workloads():
    b = load_bench()
    w = WORKLOADS["prefill_8k"]
    # 4 N (k+1) C d per head: 4 * 8192 * 17 * 64 * 128 * (4 * 32 heads)
    assert b.attention_flops(w) == 4.0 * 8192 * 17 * 64 * 128 * 128
    assert abs(b.attention_flops(w) - 5.841e11) / 5.841e11 < 1e-3
    d = WORKLOADS["decode_128k"]
    # landmarks of 2047 past chunks + K and V of 33 chunks of 64 rows, bf16, per (b, g), 128 of them
    lm = 2 * 128 * 128 * 2047
    kv = 2 * 128 * 128 * 33 * 2 * 64
    assert b.landmark_bytes(d) == lm
    assert b.decode_bytes(d) == lm + kv
    assert abs(b.decode_bytes(d) - 205.5e6) / 205.5e6 < 1e-3   # about 205 MB a decode step


def test_landmark_generation_bytes():
    b = load_bench()
    w = WORKLOADS["decode_4m_needles"]
    # per kv-head: 4,194,304 key rows of 128 bf16, then 65,536 landmark queries in and landmarks out
    # (128 bf16 each) and 65,536 float biases out; 8 kv-heads
    per_head = 4194304 * 128 * 2 + 2 * 65536 * 128 * 2 + 65536 * 4
    assert b.landmark_gen_bytes(w) == 8 * per_head
    assert abs(b.landmark_gen_bytes(w) - 8.86e9) / 8.86e9 < 1e-3


def _fake_tree(tmp_path, text):
    csrc = tmp_path / "chunk_wise_hierarchical_hils_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(text)
    (tmp_path / "profiles").mkdir()
    rec = {"kern": {"workload": "prefill_8k", "dram_bytes_per_launch": 1234,
                    "sources": {"k.cu": hashlib.sha256(b"kernel v1").hexdigest()}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    return tmp_path


@pytest.mark.parametrize("text,workload,expect", [
    ("kernel v1", "prefill_8k", 1234),     # same source, same workload
    ("kernel v2", "prefill_8k", None),     # source changed since the capture
    ("kernel v1", "decode_128k", None),    # another workload
])
def test_traffic_only_for_the_captured_sources(tmp_path, text, workload, expect):
    b = load_bench()
    b.ROOT = str(_fake_tree(tmp_path, text))
    assert b.kernel_traffic("kern", workload) == expect
    assert b.kernel_traffic("missing", workload) is None


@pytest.mark.parametrize("workload", ["tiny_f32", "decode_128k"])
def test_reference_arm_prints_one_contract_line(workload):
    """bench.py --impl reference times the oracle on the host (no GPU) and prints one JSON line with the
    contract's keys; for the small case the whole run takes seconds."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", workload], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["config"]["workload"] == workload
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["steps"] == 1
    assert line["unit"] == ("GB/s" if workload.startswith("decode") else "tokens/s")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    # under torchrun only rank 0 runs the oracle and prints; the other ranks exit 0 without work
    import subprocess
    import sys
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny_f32", "--gpus", "2"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.strip().startswith("{")]


@pytest.mark.parametrize("plan,n", [
    ("forward=two-call select=tc-heads-resident attend=union-tc", 3),
    ("forward=two-call select=tc-queries attend=chunk-major", 10),
    ("forward=two-call select=cuda-cores attend=cuda-cores", 2),
    ("forward=decode-fused select=decode-scan attend=decode-mma", 1),
    ("forward=two-call select=decode-scan attend=decode-mma", 2),
])
def test_launches_per_step_follow_the_plan(plan, n):
    """The JSON line's gpu_launches counts the library's kernels from the plan hils_describe reports."""
    b = load_bench()
    w = WORKLOADS["decode_128k"] if "decode" in plan else WORKLOADS["prefill_8k"]
    assert b.kernels_per_step(w, plan) == n


def test_traffic_entries_name_their_workload():
    """Every traffic.json entry is keyed kernel@workload, names a bench workload and lists the sources
    whose hashes gate it."""
    data = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for k, rec in data.items():
        if k.startswith("_"):
            continue
        kernel, wl = k.split("@")
        assert rec["workload"] == wl and wl in WORKLOADS
        assert rec["sources"] and rec["dram_bytes_per_launch"] > 0
