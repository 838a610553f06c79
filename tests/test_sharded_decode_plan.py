"""The exchange protocol of a sequence-sharded long decode, checked on CPU ranks (gloo) with the oracle
standing in for each rank's local compute.

Plan: the key/value and landmark caches of one sequence are split by contiguous chunk ranges over the
ranks.  For a decode query each rank
  1. scores its own chunks that lie before the query's chunk and keeps its local top-k by group score
     (equal scores: lower chunk index), with each kept chunk's per-head scores;
  2. all-gathers those k candidates (group score, chunk, G per-head scores) -- the rank owning the
     query's own chunk also contributes that chunk's per-head scores;
  3. takes the global top-k of the gathered candidates with the same rule (the global top-k lies in
     the union of the local ones), adds the own chunk, and from the gathered per-head scores the
     per-head maximum M over the selection;
  4. attends inside its own selected chunks and forms, per head, sum_c e^{s_c - M} o_c and
     sum_c e^{s_c - M};
  5. all-reduces (sum) those d + 1 numbers per head; the output is their ratio.
Every rank must end with the oracle's single-process selection and output.  No rank reads another
rank's cache: only candidate lists and per-head partial sums cross.
"""
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


def chunk_range(nL, world, rank):
    """Contiguous chunk range [lo, hi) of `rank`."""
    base, extra = divmod(nL, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def _worker(rank, world, port, out_dir, case):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from oracle import oracle as orc
    B, H, Hkv, T, d, C, k, seed = case
    G = H // Hkv
    r = np.random.default_rng(seed)
    Q = r.standard_normal((B, H, 1, d))
    K = r.standard_normal((B, Hkv, T, d))
    V = r.standard_normal((B, Hkv, T, d))
    nL = -(-T // C)
    L = r.standard_normal((B, Hkv, nL, d))
    if seed % 2:            # planted exact ties across rank boundaries: duplicate landmarks
        L[:, :, 1::3] = L[:, :, 0:1]
    scale = 1.0 / np.sqrt(d)
    pos = T - 1
    ci = pos // C
    lo, hi = chunk_range(nL, world, rank)

    def kv(b, g, c):
        t0, t1 = c * C, min(c * C + C, T)
        Kc, Vc = np.zeros((C, d)), np.zeros((C, d))
        Kc[:t1 - t0], Vc[:t1 - t0] = K[b, g, t0:t1], V[b, g, t0:t1]
        return Kc, Vc

    def local_attend(b, g, chunks):
        """Per-head scores [G, n] and per-chunk outputs [G, n, d] of this rank's chunks (the oracle)."""
        n = len(chunks)
        if n == 0:
            return np.zeros((G, 0)), np.zeros((G, 0, d))
        sel = np.array(list(chunks), dtype=np.int32)
        Ks = np.stack([kv(b, g, c)[0] for c in chunks])
        Vs = np.stack([kv(b, g, c)[1] for c in chunks])
        res = orc.attend(Q[b, g * G:(g + 1) * G, 0], sel, L[b, g, sel], Ks, Vs, C, pos, scale, want_chunks=True)
        return res["s"], res["oc"]

    O = np.zeros((B, H, d))
    SEL = np.zeros((B, Hkv, k), dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            q = Q[b, g * G:(g + 1) * G, 0]
            # 1. local candidates and local top-k
            cand = np.arange(lo, min(hi, ci))
            gs = orc.group_scores(q, L[b, g, cand], scale) if len(cand) else np.zeros(0)
            top = orc.topk(gs, len(cand), k) if len(cand) else np.full(k, -1)
            kept = [int(cand[j]) for j in top if j >= 0]
            s_kept, _ = local_attend(b, g, kept)
            msg = np.full((k, 2 + G), -np.inf)
            msg[:, 1] = -1
            for j, c in enumerate(kept):
                msg[j, 0], msg[j, 1], msg[j, 2:] = gs[list(cand).index(c)], c, s_kept[:, j]
            own = np.full(G, -np.inf)
            if lo <= ci < hi:
                own = local_attend(b, g, [ci])[0][:, 0]
            # 2. all-gather the candidates and the own chunk's scores
            t = torch.from_numpy(np.concatenate([msg.ravel(), own]))
            parts = [torch.zeros_like(t) for _ in range(world)]
            dist.all_gather(parts, t)
            allc = np.concatenate([p.numpy()[:k * (2 + G)].reshape(k, 2 + G) for p in parts])
            own_s = np.max(np.stack([p.numpy()[k * (2 + G):] for p in parts]), axis=0)
            # 3. global top-k: higher group score first, equal scores by lower chunk index
            real = allc[allc[:, 1] >= 0]
            order = sorted(range(len(real)), key=lambda j: (-real[j, 0], real[j, 1]))[:min(k, ci)]
            sel = [int(real[j, 1]) for j in order]
            SEL[b, g, :len(sel)] = sel
            SEL[b, g, len(sel):] = -1
            s_sel = np.stack([real[j, 2:] for j in order] + [own_s], axis=1)   # [G, m + 1]
            M = s_sel.max(axis=1)
            # 4. partial sums over this rank's selected chunks
            mine = [c for c in sel + [ci] if lo <= c < hi]
            s_mine, oc = local_attend(b, g, mine)
            num = np.zeros((G, d))
            den = np.zeros(G)
            for j in range(len(mine)):
                e = np.exp(s_mine[:, j] - M)
                num += e[:, None] * oc[:, j]
                den += e
            # 5. all-reduce (sum) of d + 1 numbers per head
            t = torch.from_numpy(np.concatenate([num.ravel(), den]))
            dist.all_reduce(t)
            tot = t.numpy()
            O[b, g * G:(g + 1) * G] = tot[:G * d].reshape(G, d) / tot[G * d:][:, None]
    ref = orc.forward(Q, K, V, L, C, k, q_offset=pos, scale=scale, nthreads=1)
    err = float(np.abs(O - ref["O"][:, :, 0]).max())
    same_sel = bool(np.array_equal(SEL, ref["sel"][:, :, 0, :k]))
    np.save(os.path.join(out_dir, "rank%d.npy" % rank), np.array([err, float(same_sel)]))
    dist.barrier()
    dist.destroy_process_group()


def test_chunk_ranges_partition_the_cache():
    for nL in (1, 5, 64, 65537):
        for world in (1, 2, 3, 8):
            got = []
            for rank in range(world):
                lo, hi = chunk_range(nL, world, rank)
                got += list(range(lo, hi))
            assert got == list(range(nL))


@pytest.mark.parametrize("world,case", [
    (2, (2, 4, 2, 64 * 12 + 5, 16, 16, 5, 10)),     # own chunk partial, on the last rank
    (3, (1, 6, 2, 32 * 40, 8, 32, 7, 11)),          # planted exact ties across rank boundaries
    (4, (1, 2, 1, 16 * 9, 8, 16, 12, 12)),          # k beyond the visible past: every chunk taken
])
def test_sharded_decode_matches_the_single_process_oracle(tmp_path, world, case):
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path), case), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        err, same = np.load(os.path.join(str(tmp_path), "rank%d.npy" % rank))
        assert same == 1.0, "rank %d: selection differs from the oracle's" % rank
        assert err <= 1e-12, "rank %d: output error %.3g" % (rank, err)
