#!/usr/bin/env python
"""Benchmark of the HiLS attention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl hils|reference]

One step = one pass of the whole path (landmark scoring + top-k selection, then
chunk attention + fusion) over the workload's synthetic inputs, which are
resident in HBM.  Default: prefill at training length, bf16 GQA (B=4, H=32,
Hkv=8, N=8192, d=128, C=64, k=16) as the headline, then batched decode over a
128K cache (B=16), single-token decode over a 4M cache, and prefill of a 256K
sequence with planted needles, each as a sub-record of the same line with its
own roofline, clocks, end-to-end figure and CPU baseline.  Under torchrun every rank runs
its own copy of the workload (the path has no exchange step: replicas, weak
scaling); the device time is the maximum over ranks.  Rank 0 prints one JSON
line.  ``--impl reference`` times the float64 CPU oracle instead, on bounded
samples of the same workload.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HiLS fwd tokens/s (prefill) & decode KV GB/s at 1 B200; % of tensor/HBM roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None,
                    help="one workload; default: prefill_8k (the headline) then decode_128k, decode_4m_needles "
                         "and prefill_256k_needles as sub-records of the same line")
    ap.add_argument("--impl", default="hils", choices=["hils", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--min-timed-ms", type=float, default=500.0,
                    help="decode and sub-record workloads repeat their step until the timed region lasts this "
                         "long (so that the clock sampler sees the GPU under load); 0 times exactly --steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-blocks", type=int, default=16, help="64-query blocks in the oracle sample")
    ap.add_argument("--override", nargs="*", default=[], metavar="KEY=VALUE",
                    help="change workload fields, e.g. B=4 T=524288 q_offset=524287 (smaller profiling cases)")
    ap.add_argument("--part", default="forward", choices=["forward", "landmarks", "window"],
                    help="forward: the hot path (default); landmarks: landmark generation over the "
                         "workload's whole key cache; window: the forward pass with a local window of "
                         "--window-chunks chunks and a per-chunk bias")
    ap.add_argument("--window-chunks", type=int, default=8,
                    help="window of --part window in chunks (8 x 64 = a 512-token window)")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="weak: every rank runs the whole workload; strong: the batch is split over ranks")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work per step

def attention_flops(w):
    """Nominal attention FLOPs: 4*N*(k+1)*C*d per head (QK^T and PV over k+1 chunks)."""
    return 4.0 * w.N * (w.k + 1) * w.C * w.d * w.B * w.H


def scoring_flops(w):
    """Group scores over the visible chunks (2d per query group and chunk) + per-head slot scores."""
    vis = sum((w.q_offset + i) // w.C for i in range(w.N))
    return 2.0 * w.d * vis * w.B * w.Hkv + 2.0 * w.d * (w.k + 1) * w.N * w.B * w.H


def decode_bytes(w):
    """Landmarks of the past chunks + keys and values of the k+1 selected chunks, per step (N == 1)."""
    es = 2 if w.dtype == "bf16" else 4
    ci = w.q_offset // w.C
    return es * w.B * w.Hkv * w.d * (ci + (min(w.k, ci) + 1) * 2 * w.C)


def landmark_bytes(w):
    es = 2 if w.dtype == "bf16" else 4
    return es * w.B * w.Hkv * w.d * (w.q_offset // w.C)


def landmark_gen_bytes(w):
    """Landmark generation over every chunk: the key cache and the landmark queries read once, the
    landmarks and the float biases written once."""
    es = 2 if w.dtype == "bf16" else 4
    return w.B * w.Hkv * (es * w.T * w.d + 2 * es * w.nL * w.d + 4 * w.nL)


def decode_fused_applies(w, n_sm=148):
    """Whether hils_forward runs a single-token decode as one fused kernel (bf16, d = 128, C = 64, at
    most one (b, kv-head) pair per SM, at most 4096 landmark rows per CTA)."""
    if w.N != 1 or w.dtype != "bf16" or w.d != 128 or w.C != 64 or w.G > 16 or w.k > 64:
        return False
    if os.environ.get("HILS_DECODE_FUSED") == "0":
        return False
    bg = w.B * w.Hkv
    if bg > n_sm:
        return False
    S = min(n_sm // bg, 32)
    n_past = w.q_offset // w.C if w.k > 0 else 0
    return -(-n_past // 4096) <= S


def kernels_per_step(w, plan=None):
    """Kernels of this library one step launches (the input generator, copies and memsets are not
    counted), from the library's own description of the kernels it runs for the problem."""
    if plan is None:
        import chunk_wise_hierarchical_hils_b200 as hils
        dt = {"f32": hils.HILS_F32, "bf16": hils.HILS_BF16}[w.dtype]
        plan = hils.hils_describe(hils.problem(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.k, w.q_offset, dt, dt))
    if w.N == 1:
        return 1 if "forward=decode-fused" in plan else 2   # fused kernel; or scan + top-k, attention
    n = 1                                                    # the selection
    if "attend=chunk-major" in plan:
        # V to f16; count, three scan launches, tile table, scatter; attention; finalize
        n += 9
    elif "attend=union-tc" in plan:
        n += 2                                               # V to f16; attention
    else:
        n += 1                                               # CUDA-core attention
    return n


def kernel_traffic(kernel, workload):
    """DRAM bytes per launch from an ncu capture committed in profiles/traffic.json, or None.

    Entries are keyed "kernel@workload" (or "kernel" alone).  The entry names the source files the kernel is built from with their SHA-256 at the time of the
    capture; it is used only while every one of them is unchanged, and for the same workload."""
    import hashlib
    try:
        data = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
        rec = data.get(kernel + "@" + workload) or data[kernel]
        csrc = os.path.join(ROOT, "chunk_wise_hierarchical_hils_b200", "csrc")
        for f, sha in rec["sources"].items():
            if hashlib.sha256(open(os.path.join(csrc, f), "rb").read()).hexdigest() != sha:
                return None
    except Exception:
        return None
    if rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        self.proc.wait()
        self.file.flush()
        rows = [l.split(", ") for l in open(self.file.name) if l.strip()]
        os.unlink(self.file.name)
        sm = []
        smax = None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                s, mx, pw = float(r[1]), float(r[2]), float(r[3])
            except (ValueError, IndexError):
                continue
            smax = mx
            if pw > 250.0:         # under load
                sm.append(s)
                for n, v in zip(names, r[5:9]):
                    if v.strip() == "Active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples_under_load": len(sm)}


# ---------------------------------------------------------------------------

def dist_setup(args):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def allmax(ws, vals, device="cuda"):
    """Element-wise maximum over ranks (the device time of a multi-GPU step is the slowest rank's)."""
    import torch
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    if ws > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def shard_batch(B, world, rank):
    """Contiguous slice [b0, b1) of the batch for `rank` when one problem is split over ranks.

    Sequences (and their kv-groups) are independent units of the path, so a split needs no
    exchange: every rank attends its own sequences against its own caches."""
    base, extra = divmod(B, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)


def cpu_baseline(w, n_blocks, block=64, seed=5):
    """The float64 oracle on a bounded sample: n_blocks blocks of `block` consecutive queries of batch 0.

    Returns (value in the workload's unit, cores, description, seconds of oracle time)."""
    import numpy as np
    from oracle import oracle as orc
    from synth import workloads as W
    cores = orc.max_threads()
    rng = np.random.default_rng(seed)
    if w.N == 1:
        # decode: a bounded number of (b, g) query groups, every one a full decode of its sequence
        n_groups = min(w.B * w.Hkv, max(1, n_blocks // 4))
        items = [(b, g) for b in range(w.B) for g in range(w.Hkv)][:n_groups]
        t = 0.0
        ci = w.q_offset // w.C
        for (b, g) in items:
            Lr, _ = W.l_rows(w, b, g, 0, ci + 1)
            q, _ = W.q_rows(w, b, np.arange(g * w.G, (g + 1) * w.G), np.array([0]))
            sel_c = None
            t0 = time.perf_counter()
            sel, _ = orc.select(q[:, 0], Lr, w.C, w.k, w.q_offset, orc.default_scale(w.d))
            t += time.perf_counter() - t0
            sel_c = [int(c) for c in sel if c >= 0]
            Ls = np.zeros((w.k + 1, w.d))
            Ks = np.zeros((w.k + 1, w.C, w.d))
            Vs = np.zeros((w.k + 1, w.C, w.d))
            for j, c in enumerate(sel):
                if c < 0:
                    continue
                t0_, t1_ = c * w.C, min((c + 1) * w.C, w.T)
                Ks[j, :t1_ - t0_] = W.k_rows(w, b, g, t0_, t1_)[0]
                Vs[j, :t1_ - t0_] = W.v_rows(w, b, g, t0_, t1_)[0]
                Ls[j] = Lr[c]
            t0 = time.perf_counter()
            orc.attend(q[:, 0], sel, Ls, Ks, Vs, w.C, w.q_offset, orc.default_scale(w.d))
            t += time.perf_counter() - t0
        per_group_bytes = decode_bytes(w) / (w.B * w.Hkv)
        return (per_group_bytes * len(items) / t / 1e9, 1,
                "%d of %d decode query groups (b, kv-head), one thread each, host input generation untimed"
                % (len(items), w.B * w.Hkv), t)
    if w.T > 32768:
        # a long sequence: sampled query groups (b, kv-head, query), each scored over all its visible
        # chunks and attended over its selection, one thread; only the rows a group needs are generated
        n_groups = max(8, 2 * n_blocks)
        items = sorted((int(rng.integers(0, w.B)), int(rng.integers(0, w.Hkv)), int(rng.integers(0, w.N)))
                       for _ in range(n_groups))
        scale = orc.default_scale(w.d)
        lrows = {}
        t = 0.0
        for (b, g, i) in items:
            pos = w.q_offset + i
            ci = pos // w.C
            if (b, g) not in lrows or lrows[(b, g)].shape[0] <= ci:
                lrows[(b, g)] = W.l_rows(w, b, g, 0, w.nL)[0]
            Lr = lrows[(b, g)]
            q, _ = W.q_rows(w, b, np.arange(g * w.G, (g + 1) * w.G), np.array([i]))
            t0 = time.perf_counter()
            sel, _ = orc.select(q[:, 0], Lr, w.C, w.k, pos, scale)
            t += time.perf_counter() - t0
            Ls = np.zeros((w.k + 1, w.d))
            Ks = np.zeros((w.k + 1, w.C, w.d))
            Vs = np.zeros((w.k + 1, w.C, w.d))
            for j, c in enumerate(sel):
                if c < 0:
                    continue
                r0, r1 = c * w.C, min((c + 1) * w.C, w.T)
                Ks[j, :r1 - r0] = W.k_rows(w, b, g, r0, r1)[0]
                Vs[j, :r1 - r0] = W.v_rows(w, b, g, r0, r1)[0]
                Ls[j] = Lr[c]
            t0 = time.perf_counter()
            orc.attend(q[:, 0], sel, Ls, Ks, Vs, w.C, pos, scale)
            t += time.perf_counter() - t0
        return (len(items) / w.Hkv / t, 1,
                "%d query groups (b, kv-head, query) at random positions, one thread each (a token is Hkv "
                "query groups), host input generation untimed" % len(items), t)
    b = 0
    K = np.stack([W.k_rows(w, b, g, 0, w.T)[0] for g in range(w.Hkv)])[None]
    V = np.stack([W.v_rows(w, b, g, 0, w.T)[0] for g in range(w.Hkv)])[None]
    L = np.stack([W.l_rows(w, b, g, 0, w.nL)[0] for g in range(w.Hkv)])[None]
    starts = sorted(set(int(x) for x in rng.integers(0, (w.N - block) // block + 1, size=n_blocks) * block))
    t = 0.0
    ntok = 0
    for i0 in starts:
        Qb, _ = W.q_rows(w, b, np.arange(w.H), np.arange(i0, i0 + block))
        t0 = time.perf_counter()
        orc.forward(Qb[None], K, V, L, w.C, w.k, q_offset=w.q_offset + i0, nthreads=cores)
        t += time.perf_counter() - t0
        ntok += block
    return (ntok / t, cores, "%d blocks of %d consecutive queries (all %d heads) of batch 0 at random offsets; "
            "OpenMP over query groups; host input generation untimed" % (len(starts), block, w.H), t)


def run_reference(args, w):
    ws, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    unit = "tokens/s" if w.N > 1 else "GB/s"
    vals, secs = [], []
    for s in range(args.warmup + args.steps):
        v, cores, desc, t = cpu_baseline(w, n_blocks=2, seed=100 + s)
        if s >= args.warmup:
            vals.append(v)
            secs.append(t)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def config_of(w, n):
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "T": w.T, "d": w.d, "C": w.C,
            "k": w.k, "q_offset": w.q_offset, "dtype_in": w.dtype, "dtype_out": w.dtype,
            "parallelism": "replicas x%d (no exchange step)" % n,
            "l2": ("L2 flushed before every timed step (%d MB written outside the timed events)" % (FLUSH_BYTES >> 20)
                   if needs_flush(w) else "inputs larger than L2 (no flush)")}


L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 256 * 1024 * 1024     # written before each timed step when a step's inputs are near L2's size
TENSOR_SPEC_TFLOPS = 2250.0         # B200 dense bf16, nominal
HBM_SPEC_GBS = 8000.0               # B200 HBM3e, nominal


def needs_flush(w):
    """Whether a step's own input bytes are small enough that replays could hit L2: decode reads only the
    landmarks and the selected chunks (about 1.2-1.6x L2), so those steps get an L2 flush before each."""
    return w.N == 1


class StepTimer:
    """Device time of graph replays with CUDA events on the replay stream.

    Without a flush: one pair of events around n back-to-back replays.  With a flush: a buffer larger
    than L2 is written before every replay, outside that replay's pair of events, and the pairs are
    summed, so that no step reads what the previous one left in L2."""

    def __init__(self, flush):
        import torch
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda") if flush else None

    def run(self, graph, n):
        import torch
        stream = torch.cuda.current_stream()
        if self.flush is None:
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                graph.replay()
            z.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(z)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, z in evs:
            self.flush.zero_()
            a.record(stream)
            graph.replay()
            z.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(z) for a, z in evs)


def tensor_peak(pk, pk_kind, timed_s):
    """The measured bf16 peak that applies: the burst figure for a timed region under a second, the
    sustained (power-capped) one for a longer region."""
    if timed_s >= 1.0 and "bf16_tflops_sustained" in pk:
        return pk["bf16_tflops_sustained"], pk_kind + " bf16 sustained (timed region %.2f s)" % timed_s
    return pk["bf16_tflops"], pk_kind + " bf16 burst (timed region %.2f s)" % timed_s


def measure_forward(args, w, ws, rank, local, steps=None):
    """One workload of the forward path: device-timed steps, per-call times, roofline of the dominant
    kernel, end to end through hils_forward with host buffers, and (rank 0, one GPU) the oracle's CPU
    baseline.  Returns the record (a dict of the JSON line's fields)."""
    import torch
    import chunk_wise_hierarchical_hils_b200 as hils
    from synth import gpu as synth_gpu

    steps = args.steps if steps is None else steps
    full_B = w.B
    if args.scaling == "strong" and ws > 1:
        b0, b1 = shard_batch(w.B, ws, rank)
        if b1 - b0 < 1:
            raise SystemExit("strong scaling needs B >= number of ranks")
        w = w.with_(B=b1 - b0, seed=w.seed * 1000 + b0)
    dev = synth_gpu.alloc_inputs(w)
    dt = {"f32": hils.HILS_F32, "bf16": hils.HILS_BF16}[w.dtype]
    p = hils.problem(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.k, w.q_offset, dt, dt)
    tdt = dev["Q"].dtype
    O = torch.empty((w.B, w.H, w.N, w.d), dtype=tdt, device="cuda")
    sel_idx = torch.empty((w.B, w.Hkv, w.N, max(w.k, 1)), dtype=torch.int32, device="cuda")
    sel_score = torch.empty((w.B, w.H, w.N, w.k + 1), dtype=torch.float32, device="cuda")
    ws_sel = torch.empty(max(hils.hils_score_select_workspace_size(p), 16), dtype=torch.uint8, device="cuda")
    ws_att = torch.empty(max(hils.hils_chunk_attend_fuse_workspace_size(p), 16), dtype=torch.uint8, device="cuda")
    ws_fwd = torch.empty(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    plan = hils.hils_describe(p)   # the kernels the library runs for this problem
    # Timing: every timed region replays a CUDA graph of the library calls (captured once after
    # warm-up), so the device times below are the kernels' and not the host's launch gaps.
    # The step graph times the whole path; a graph per call gives each call's average duration.
    def call_select():
        hils.hils_score_select(p, dev["Q"], dev["L"], sel_idx, sel_score, ws_sel)

    def call_attend():
        hils.hils_chunk_attend_fuse(p, dev["Q"], dev["K"], dev["V"], sel_idx, sel_score, O, ws_att)

    def step():
        # the public call: selection then attention (single-token decode: one fused kernel where it applies)
        hils.hils_forward(p, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws_fwd)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hils.hils_sync_status() != hils.HILS_OK:
        raise RuntimeError("device-side timeout during warm-up")

    def capture(fn):
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_):
            fn()
        return g_

    g_step = capture(step)
    # per-call graphs: prefill's selection and attention; decode's two-kernel path for comparison
    g_sel, g_att = capture(call_select), capture(call_attend)
    flush = needs_flush(w)
    timer = StepTimer(flush)
    # short steps are repeated so that the clock sampler sees the GPU under load (about half a second)
    timer.run(g_step, 2)
    probe_ms = timer.run(g_step, 4) / 4
    if (steps is None or w.N == 1) and args.min_timed_ms > 0:
        steps = max(steps or args.steps, int(args.min_timed_ms / max(probe_ms + (0.05 if flush else 0.0), 1e-3)))
    steps = steps or args.steps
    sampler = ClockSampler(local)
    barrier(ws)
    torch.cuda.synchronize()
    sampler.start()
    total_ms = timer.run(g_step, steps)
    barrier(ws)
    clocks = sampler.stop()
    n_call = min(steps, max(args.steps, 50))
    timer.run(g_sel, 2)
    k1_avg = timer.run(g_sel, n_call) / n_call
    timer.run(g_att, 2)
    k2_avg = timer.run(g_att, n_call) / n_call
    if hils.hils_sync_status() != hils.HILS_OK:
        raise RuntimeError("device-side timeout")
    total_ms, k1_avg, k2_avg = allmax(ws, [total_ms, k1_avg, k2_avg])
    ms_step = total_ms / steps
    del g_step, g_sel, g_att, timer

    # end to end through the public call with host buffers
    # prefill: every input crosses PCIe each step; decode: only the new query token does (the key/value
    # and landmark caches are state that stays resident across decode steps)
    e2e_names = ["Q", "K", "V", "L"] if w.N > 1 else ["Q"]
    pin = {}
    for k in e2e_names:
        pin[k] = torch.empty(dev[k].shape, dtype=dev[k].dtype, pin_memory=True)
        pin[k].copy_(dev[k])
    Oh = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = Oh.numel() * Oh.element_size()
    stream = torch.cuda.current_stream()
    if w.N > 1:
        # prefill: the public host-buffer call, which slices the batch by (b, kv-group) pairs and overlaps
        # each slice's copies in, forward and copy out
        ws_host = torch.empty(hils.hils_forward_host_workspace_size(p), dtype=torch.uint8, device="cuda")

        def e2e_step():
            hils.hils_forward_host(p, pin["Q"], pin["K"], pin["V"], pin["L"], Oh, ws_host, stream)
    else:
        # decode: the new token in, its output out, the caches resident
        def e2e_step():
            for k in e2e_names:
                dev[k].copy_(pin[k], non_blocking=True)
            hils.hils_forward(p, dev["Q"], dev["K"], dev["V"], dev["L"], O, ws_fwd)
            Oh.copy_(O, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    e2e_steps = args.e2e_steps if (w.N > 1 or args.min_timed_ms <= 0) else max(args.e2e_steps, 100)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allmax(ws, [e0.elapsed_time(e1) / e2e_steps])[0]
    if hils.hils_sync_status(stream) != hils.HILS_OK:
        raise RuntimeError("device-side timeout")
    del dev, O, sel_idx, sel_score, ws_sel, ws_att, ws_fwd, pin, Oh
    if w.N > 1:
        del ws_host
    torch.cuda.empty_cache()

    pk, pk_kind = peaks()
    timed_s = total_ms * 1e-3
    fused = w.N == 1 and decode_fused_applies(w)
    if w.N > 1:
        unit = "tokens/s"
        per_step_units = w.B * w.N
        fl = attention_flops(w)
        if w.dtype == "f32":
            # float32 problems run on the CUDA-core kernels: no tensor-core roofline applies; the bf16
            # figure is kept as the reference denominator and labelled so
            peak, kind = pk["bf16_tflops"], pk_kind + " bf16 burst (float32 inputs run on CUDA cores)"
        else:
            peak, kind = tensor_peak(pk, pk_kind, timed_s)
        achieved = fl / (k2_avg * 1e-3) / 1e12
        cm = "attend=chunk-major" in plan
        roof = {"bound": "tensor", "kernel": "chunk_attend_fuse (prefill, %s)" % ("chunk-major" if cm else "union"),
                "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "frac_of_spec": achieved / TENSOR_SPEC_TFLOPS,
                "traffic": kernel_traffic("attend_prefill_cm" if cm else "attend_prefill_tc", w.name),
                "peak_kind": kind,
                "algorithmic_flops_per_launch": fl, "launch_ms": k2_avg, "select_ms": k1_avg,
                "step_tflops": (fl + scoring_flops(w)) / (ms_step * 1e-3) / 1e12}
    elif fused:
        # one kernel per step (plus a memset of its tickets): its roofline is the step's bytes over the step
        unit = "GB/s"
        per_step_units = decode_bytes(w) / 1e9
        peak = pk["hbm_gbs"]
        step_gbs = decode_bytes(w) / (ms_step * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": "decode_fused (selection + attention, one cooperative kernel)",
                "achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                "traffic": kernel_traffic("decode_fused", w.name), "algorithmic_bytes_per_launch": decode_bytes(w),
                "launch_ms": ms_step, "two_kernel_select_ms": k1_avg, "two_kernel_attend_ms": k2_avg,
                "peak_kind": pk_kind + " copy", "frac_of_spec": step_gbs / HBM_SPEC_GBS, "step_gbs": step_gbs,
                "step_frac": step_gbs / peak, "step_frac_of_spec": step_gbs / HBM_SPEC_GBS}
    else:
        unit = "GB/s"
        per_step_units = decode_bytes(w) / 1e9
        lb = landmark_bytes(w)
        kvb = decode_bytes(w) - lb
        peak = pk["hbm_gbs"]
        step_gbs = decode_bytes(w) / (ms_step * 1e-3) / 1e9
        if k2_avg >= k1_avg:   # the dominant kernel: chunk attention (selected K/V) or the landmark scan
            achieved = kvb / (k2_avg * 1e-3) / 1e9
            roof = {"bound": "hbm", "kernel": "chunk_attend_fuse (decode)", "achieved": achieved, "peak": peak,
                    "unit": "GB/s", "frac": achieved / peak, "traffic": kernel_traffic("attend_decode", w.name),
                    "algorithmic_bytes_per_launch": kvb, "launch_ms": k2_avg, "select_ms": k1_avg}
        else:
            achieved = lb / (k1_avg * 1e-3) / 1e9
            roof = {"bound": "hbm", "kernel": "score_select (decode landmark scan)", "achieved": achieved,
                    "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": kernel_traffic("select_decode", w.name),
                    "algorithmic_bytes_per_launch": lb, "launch_ms": k1_avg, "attend_ms": k2_avg}
        roof.update({"peak_kind": pk_kind + " copy", "frac_of_spec": achieved / HBM_SPEC_GBS,
                     "step_gbs": step_gbs, "step_frac": step_gbs / peak, "step_frac_of_spec": step_gbs / HBM_SPEC_GBS})
    roof["plan"] = plan
    units_all = ws * per_step_units
    if args.scaling == "strong" and ws > 1:
        units_all = per_step_units * full_B / w.B   # ranks hold slices of one batch (equal slices assumed)
    rec = {"value": units_all / (ms_step * 1e-3), "unit": unit, "n_gpus": ws, "steps": steps,
           "warmup": args.warmup, "ms_per_step": ms_step, "dtype": w.dtype, "config": config_of(w, ws),
           "roofline": roof,
           "e2e": {"value": units_all / (e2e_ms * 1e-3), "unit": unit, "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
                   "inputs_copied": e2e_names,
                   "call": "hils_forward_host (pinned host buffers)" if w.N > 1 else
                           "query token H2D, hils_forward on the resident caches, output D2H"},
           "gpu_launches": kernels_per_step(w, plan) * steps, "clocks": clocks}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, cores, desc, _ = cpu_baseline(w, args.cpu_blocks)
        rec["cpu_baseline"] = {"value": v, "unit": unit, "cores": cores, "kind": "oracle", "sample": desc}
    return rec


DEFAULT_SET = ("prefill_8k", "decode_128k", "decode_4m_needles", "prefill_256k_needles")


def run_hils(args, workloads):
    """The forward path on each workload in turn; rank 0 prints one JSON line: the first workload's
    record at the top level (the headline), the others under "workloads"."""
    ws, rank, local = dist_setup(args)
    recs = []
    for n, w in enumerate(workloads):
        recs.append(measure_forward(args, w, ws, rank, local, steps=args.steps if n == 0 else None))
    head = recs[0]
    line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": ws, "steps": head["steps"],
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
            "scaling": args.scaling, "vs_baseline": None, "dtype": head["dtype"],
            "data": "synthetic (seeded Philox4x32-10 inputs)"}
    for k in ("config", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        if k in head:
            line[k] = head[k]
    line["timing"] = ("CUDA-graph replays of the library calls, CUDA events on the replay stream; decode "
                      "steps each after an L2 flush that is outside the timed events")
    if len(recs) > 1:
        line["workloads"] = {r["config"]["workload"]: r for r in recs[1:]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def timed_graph_replays(call, args, ws, local):
    """Warm up `call`, capture it in a CUDA graph and time args.steps replays with CUDA events on the
    replay stream, barriers and clock sampling around them.  Returns (ms per replay, max over ranks;
    clock record)."""
    import torch
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local)
    barrier(ws)
    torch.cuda.synchronize()
    sampler.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        graph.replay()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clocks = sampler.stop()
    ms = allmax(ws, [start.elapsed_time(end) / args.steps])[0]
    del graph
    return ms, clocks


def run_landmarks(args, w):
    """Landmark generation (hils_landmarks) over the workload's whole key cache, one call per step.

    The landmark queries are the workload's landmark tensor (seeded synthetic values of the same shape);
    the metric is algorithmic bytes per second against the measured copy bandwidth."""
    import torch
    import chunk_wise_hierarchical_hils_b200 as hils
    from synth import gpu as synth_gpu

    ws, rank, local = dist_setup(args)
    dev = synth_gpu.alloc_inputs(w)
    del dev["Q"], dev["V"]
    dt = {"f32": hils.HILS_F32, "bf16": hils.HILS_BF16}[w.dtype]
    p = hils.problem(w.B, 1, w.Hkv, 1, w.T, w.d, w.C, 0, 0, dt, dt)
    K, U = dev["K"], dev["L"]
    Lout = torch.empty_like(U)
    beta = torch.empty((w.B, w.Hkv, w.nL), dtype=torch.float32, device="cuda")
    nbytes = landmark_gen_bytes(w)

    def call():
        hils.hils_landmarks(p, K, U, Lout, beta)

    ms, clocks = timed_graph_replays(call, args, ws, local)
    if hils.hils_sync_status() != hils.HILS_OK:
        raise RuntimeError("device-side failure")
    stream = torch.cuda.current_stream()

    # end to end: keys and landmark queries from pinned host memory, landmarks and biases back
    # pinned buffers allocated directly (a 4M-token key cache is 8.6 GB: no pageable intermediate copy)
    Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
    Uh = torch.empty(U.shape, dtype=U.dtype, pin_memory=True)
    Kh.copy_(K)
    Uh.copy_(U)
    Lh = torch.empty(Lout.shape, dtype=Lout.dtype, pin_memory=True)
    bh = torch.empty(beta.shape, dtype=beta.dtype, pin_memory=True)

    def e2e_step():
        K.copy_(Kh, non_blocking=True)
        U.copy_(Uh, non_blocking=True)
        call()
        Lh.copy_(Lout, non_blocking=True)
        bh.copy_(beta, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allmax(ws, [e0.elapsed_time(e1) / args.e2e_steps])[0]

    pk, pk_kind = peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    value = ws * achieved
    line = {"metric": "HiLS landmark generation GB/s at 1 B200; % of HBM roofline", "value": value,
            "unit": "GB/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded Philox4x32-10 inputs)", "config": dict(config_of(w, ws), part="landmarks"),
            "roofline": {"bound": "hbm", "kernel": "landmarks", "achieved": achieved, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": None,
                         "peak_kind": pk_kind + " copy", "algorithmic_bytes_per_launch": nbytes,
                         "launch_ms": ms},
            "e2e": {"value": ws * nbytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": Kh.numel() * Kh.element_size() + Uh.numel() * Uh.element_size(),
                    "d2h_bytes_per_step": Lh.numel() * Lh.element_size() + bh.numel() * 4, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps, "clocks": clocks,
            "timing": "CUDA-graph replays of one hils_landmarks call, CUDA events on the replay stream"}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        from oracle import oracle as orc
        n = min(w.nL, 4096)                      # a bounded slice: the first n chunks of (b, g) = (0, 0)
        K64 = K[0:1, 0:1, :min(w.T, n * w.C)].double().cpu().numpy()
        U64 = U[0:1, 0:1, :n].double().cpu().numpy()
        t0 = time.perf_counter()
        orc.landmarks(K64, U64, w.C)
        t = time.perf_counter() - t0
        es = 2 if w.dtype == "bf16" else 4
        line["cpu_baseline"] = {"value": (K64.size + 2 * U64.size) * es / t / 1e9, "unit": "GB/s", "cores": 1,
                                "kind": "oracle", "sample": "%d chunks of one (b, kv-head), one thread" % n}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_window(args, w):
    """The forward pass with a local window and a per-chunk bias (hils_forward_window), one call per step.

    Algorithmic work: the attention FLOPs over k + wc slots per query (nominal, as for the plain path)."""
    import numpy as np
    import torch
    import chunk_wise_hierarchical_hils_b200 as hils
    from synth import gpu as synth_gpu

    ws, rank, local = dist_setup(args)
    wc = args.window_chunks
    dev = synth_gpu.alloc_inputs(w)
    dt = {"f32": hils.HILS_F32, "bf16": hils.HILS_BF16}[w.dtype]
    p = hils.problem(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.k, w.q_offset, dt, dt)
    bias = torch.from_numpy(np.random.default_rng(w.seed + 7).standard_normal((w.B, w.Hkv, w.nL))
                            .astype(np.float32)).cuda()
    O = torch.empty((w.B, w.H, w.N, w.d), dtype=dev["Q"].dtype, device="cuda")
    wsp = torch.empty(hils.hils_forward_window_workspace_size(p, wc), dtype=torch.uint8, device="cuda")

    def call():
        hils.hils_forward_window(p, wc, bias, dev["Q"], dev["K"], dev["V"], dev["L"], O, wsp)

    ms, clocks = timed_graph_replays(call, args, ws, local)
    if hils.hils_sync_status() != hils.HILS_OK:
        raise RuntimeError("device-side failure")
    pk, pk_kind = peaks()
    wk = w.with_(k=w.k + wc - 1)
    fl = attention_flops(wk)
    peak, peak_kind = tensor_peak(pk, pk_kind, ms * 1e-3 * args.steps)
    achieved = fl / (ms * 1e-3) / 1e12
    units = w.B * w.N if w.N > 1 else w.B
    line = {"metric": "HiLS fwd with a %d-chunk local window and chunk bias, tokens/s at 1 B200" % wc,
            "value": ws * units / (ms * 1e-3), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded Philox4x32-10 inputs)",
            "config": dict(config_of(w, ws), part="window", window_chunks=wc),
            "roofline": {"bound": "tensor", "kernel": "whole step (selection + attention)", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                         "peak_kind": peak_kind, "algorithmic_flops_per_launch": fl},
            "gpu_launches": kernels_per_step(w) * args.steps, "clocks": clocks,
            "timing": "CUDA-graph replays of one hils_forward_window call, CUDA events on the replay stream"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    args = parse()
    from synth.workloads import WORKLOADS
    names = [args.workload] if args.workload else list(DEFAULT_SET)
    if args.impl == "reference" or args.part != "forward" or args.override:
        names = names[:1]
    w = WORKLOADS[names[0]]
    if args.override:
        kv = dict(x.split("=", 1) for x in args.override)
        w = w.with_(**{k: type(getattr(w, k))(v) for k, v in kv.items()})
        w = w.with_(name=w.name + "[" + ",".join(args.override) + "]")
    if args.impl == "reference" and args.part != "forward":
        raise SystemExit("--part %s times the library only; the reference arm covers the forward path" % args.part)
    if args.impl == "reference":
        run_reference(args, w)
    elif args.part == "landmarks":
        run_landmarks(args, w)
    elif args.part == "window":
        run_window(args, w)
    else:
        run_hils(args, [w] + [WORKLOADS[n] for n in names[1:]])


if __name__ == "__main__":
    main()
