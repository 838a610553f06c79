"""Multi-rank host logic on CPU (gloo, world size 2): batch sharding without an
exchange step reproduces the single-rank result, and timings reduce to the
slowest rank."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from oracle import oracle as orc
    from synth import workloads as W
    from synth.workloads import Workload
    w = Workload("shard", B=3, H=4, Hkv=2, N=96, T=96, d=16, C=8, k=3, q_offset=0, dtype="f32", seed=3,
                 l_mode="chunkmean")
    b0, b1 = bench.shard_batch(w.B, world, rank)
    inp = W.full_inputs(w)
    sl = {k: v[0][b0:b1] for k, v in inp.items()}
    res = orc.forward(sl["Q"], sl["K"], sl["V"], sl["L"], w.C, w.k, nthreads=1)
    # gather the shards (variable batch sizes: pad to the largest slice)
    pad = np.zeros((w.B - (w.B // world) * (world - 1) + 1, w.H, w.N, w.d))
    pad[:b1 - b0] = res["O"]
    t = torch.from_numpy(pad)
    parts = [torch.zeros_like(t) for _ in range(world)]
    dist.all_gather(parts, t)
    slowest = bench.allmax(world, [float(rank + 1), 10.0 - rank], device="cpu")
    if rank == 0:
        got = np.concatenate([parts[r].numpy()[:bench.shard_batch(w.B, world, r)[1] - bench.shard_batch(w.B, world, r)[0]]
                              for r in range(world)])
        full = orc.forward(*(inp[k][0] for k in ("Q", "K", "V", "L")), w.C, w.k, nthreads=1)["O"]
        np.save(os.path.join(out_dir, "err.npy"), np.array([np.abs(got - full).max()] + slowest))
    dist.barrier()
    dist.destroy_process_group()


def test_shards_cover_batch_exactly_once():
    import bench
    for B in (1, 2, 3, 7, 16):
        for world in (1, 2, 4):
            cover = []
            for r in range(world):
                b0, b1 = bench.shard_batch(B, world, r)
                cover += list(range(b0, b1))
            assert cover == list(range(B))


def test_two_rank_gloo_matches_single(tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    err = np.load(tmp_path / "err.npy")
    assert err[0] <= 1e-15
    assert list(err[1:]) == [2.0, 10.0]
