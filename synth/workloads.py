"""Seeded synthetic workloads for HiLS attention (host side, numpy).

Each workload fixes shapes and a value recipe.  Every input value is a pure
function of (seed, stream, flat index), so any slice can be rebuilt on its own:
the oracle asks for exactly the rows it needs, the GPU side fills whole tensors
with the CUDA twin of this module (``synth/gen_cuda.cu``).

Value recipe (all deviates from :func:`synth.philox.gaussian_at`):

* ``Q[b,h,i,:]`` stream 1, ``K`` stream 2, ``V`` stream 3, landmarks ``L`` stream 4.
* ``l_mode == "chunkmean"``: ``L[b,g,c,:]`` is the float64 mean (rows summed in
  order) of the chunk's *rounded* key rows plus ``l_noise`` times a deviate of
  stream 5.
* needles: one unit vector ``u_g`` per kv-head (stream 6, normalised with a
  sequential sum of squares); ``n_needles`` chunks per kv-head, one drawn
  uniformly inside each of ``n_needles`` equal strata of the chunk range
  (stream 7).  Keys of a needle chunk and its landmark get ``+shift*u_g``;
  queries at positions ``p % needle_period == 0`` get ``+shift*u_{h//G}``.
* rounding: the float64 value is rounded once to float32 (nearest-even), and
  for bf16 workloads that float32 once more to bfloat16 (nearest-even).

The module contains no attention arithmetic.
"""
from dataclasses import dataclass, replace
import math
import numpy as np

from .philox import gaussian_at, uniform_at, f64_to_f32, f32_to_bf16_bits, bf16_bits_to_f64

S_Q, S_K, S_V, S_L, S_LNOISE, S_U, S_NEEDLE = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int          # queries
    T: int          # kv length
    d: int
    C: int
    k: int
    q_offset: int
    dtype: str      # "f32" | "bf16"
    seed: int
    input_scale: bool = False   # multiply every deviate by d**-0.25
    l_mode: str = "iid"         # "iid" | "chunkmean"
    l_noise: float = 0.1
    n_needles: int = 0
    needle_period: int = 0
    needle_shift: float = 3.0

    @property
    def G(self):
        return self.H // self.Hkv

    @property
    def nL(self):
        return -(-self.T // self.C)

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    # tiny fp32 prefill: i.i.d. N(0,1) * d^-1/4, seed 0
    "tiny_f32": Workload("tiny_f32", B=1, H=2, Hkv=2, N=1024, T=1024, d=64, C=32, k=4,
                         q_offset=0, dtype="f32", seed=0, input_scale=True),
    # prefill at training length, bf16 GQA, landmarks = chunk mean of keys + N(0, 0.1^2)
    "prefill_8k": Workload("prefill_8k", B=4, H=32, Hkv=8, N=8192, T=8192, d=128, C=64, k=16,
                           q_offset=0, dtype="bf16", seed=1, l_mode="chunkmean"),
    # long prefill with planted needle chunks
    "prefill_256k_needles": Workload("prefill_256k_needles", B=1, H=16, Hkv=4, N=262144, T=262144,
                                     d=128, C=64, k=32, q_offset=0, dtype="bf16", seed=2,
                                     n_needles=64, needle_period=512),
    # batched single-token decode over a 128K cache
    "decode_128k": Workload("decode_128k", B=16, H=32, Hkv=8, N=1, T=131072, d=128, C=64, k=32,
                            q_offset=131071, dtype="bf16", seed=3, l_mode="chunkmean"),
    # single-token decode over a 4M cache with planted needles
    "decode_4m_needles": Workload("decode_4m_needles", B=1, H=32, Hkv=8, N=1, T=4194304, d=128,
                                  C=64, k=64, q_offset=4194303, dtype="bf16", seed=4,
                                  n_needles=16, needle_period=512),
}


def _round(w, v64):
    """float64 values -> (float64 exact view of the rounded value, raw array for upload)."""
    f32 = f64_to_f32(v64)
    if w.dtype == "f32":
        return f32.astype(np.float64), f32
    bits = f32_to_bf16_bits(f32)
    return bf16_bits_to_f64(bits), bits


def _scale(w):
    # d**-0.25 as 1/sqrt(sqrt(d)): IEEE sqrt and division are correctly rounded on every platform
    return 1.0 / math.sqrt(math.sqrt(w.d)) if w.input_scale else 1.0


def needle_u(w, g):
    """Unit vector u_g (float64, length d) for kv-head g."""
    z = gaussian_at(w.seed, S_U, np.arange(g * w.d, (g + 1) * w.d, dtype=np.uint64))
    ss = 0.0
    for x in z:                 # sequential sum of squares (the CUDA twin uses the same order)
        ss = ss + x * x
    return z / math.sqrt(ss)


def needle_chunks(w, g):
    """Sorted needle chunk indices of kv-head g (empty without needles)."""
    if not w.n_needles:
        return np.zeros(0, dtype=np.int64)
    width = (w.T // w.C) // w.n_needles
    m = np.arange(w.n_needles, dtype=np.uint64)
    u = uniform_at(w.seed, S_NEEDLE, np.uint64(g * w.n_needles) + m)
    off = np.floor(u * width).astype(np.int64)
    return np.arange(w.n_needles, dtype=np.int64) * width + off


def _flat(shape, idx_tuple):
    """Row-major flat index (uint64) of a broadcast index tuple."""
    e = np.zeros(np.broadcast(*idx_tuple).shape, dtype=np.uint64)
    for n, ix in zip(shape, idx_tuple):
        e = e * np.uint64(n) + np.asarray(ix, dtype=np.uint64)
    return e


def q_rows(w, b, heads, pos_idx):
    """Q[b, heads, pos_idx, :] -> (float64 [len(heads), len(pos_idx), d], raw)."""
    heads = np.asarray(heads, dtype=np.int64)
    pos_idx = np.asarray(pos_idx, dtype=np.int64)
    e = _flat((w.B, w.H, w.N, w.d), (b, heads[:, None, None], pos_idx[None, :, None],
                                     np.arange(w.d)[None, None, :]))
    v = gaussian_at(w.seed, S_Q, e) * _scale(w)
    if w.n_needles:
        hit = ((w.q_offset + pos_idx) % w.needle_period) == 0
        if hit.any():
            for a, h in enumerate(heads):
                u = needle_u(w, int(h) // w.G)
                v[a, hit, :] = v[a, hit, :] + w.needle_shift * u[None, :]
    return _round(w, v)


def _kv_raw64(w, stream, b, g, t0, t1):
    t = np.arange(t0, t1, dtype=np.int64)
    e = _flat((w.B, w.Hkv, w.T, w.d), (b, g, t[:, None], np.arange(w.d)[None, :]))
    v = gaussian_at(w.seed, stream, e) * _scale(w)
    if stream == S_K and w.n_needles:
        nc = needle_chunks(w, g)
        hit = np.isin(t // w.C, nc)
        if hit.any():
            v[hit, :] = v[hit, :] + w.needle_shift * needle_u(w, g)[None, :]
    return v


def k_rows(w, b, g, t0, t1):
    """K[b, g, t0:t1, :] -> (float64 [t1-t0, d], raw)."""
    return _round(w, _kv_raw64(w, S_K, b, g, t0, t1))


def v_rows(w, b, g, t0, t1):
    return _round(w, _kv_raw64(w, S_V, b, g, t0, t1))


def l_rows(w, b, g, c0, c1):
    """L[b, g, c0:c1, :] -> (float64 [c1-c0, d], raw)."""
    c = np.arange(c0, c1, dtype=np.int64)
    if w.l_mode == "chunkmean":
        out = np.empty((c1 - c0, w.d), dtype=np.float64)
        kk, _ = k_rows(w, b, g, c0 * w.C, min(c1 * w.C, w.T))
        for a, cc in enumerate(c):
            r0 = (cc - c0) * w.C
            rows = kk[r0:r0 + min(w.C, w.T - cc * w.C)]
            acc = rows[0].copy()
            for r in range(1, rows.shape[0]):      # sequential float64 sum
                acc = acc + rows[r]
            out[a] = acc / rows.shape[0]
        e = _flat((w.B, w.Hkv, w.nL, w.d), (b, g, c[:, None], np.arange(w.d)[None, :]))
        v = out + w.l_noise * gaussian_at(w.seed, S_LNOISE, e)
        return _round(w, v)
    e = _flat((w.B, w.Hkv, w.nL, w.d), (b, g, c[:, None], np.arange(w.d)[None, :]))
    v = gaussian_at(w.seed, S_L, e) * _scale(w)
    if w.n_needles:
        hit = np.isin(c, needle_chunks(w, g))
        if hit.any():
            v[hit, :] = v[hit, :] + w.needle_shift * needle_u(w, g)[None, :]
    return _round(w, v)


def full_inputs(w):
    """Whole tensors for small workloads: dict name -> (float64 array, raw array).

    Shapes: Q [B,H,N,d], K/V [B,Hkv,T,d], L [B,Hkv,nL,d].
    """
    Q64 = np.empty((w.B, w.H, w.N, w.d))
    K64 = np.empty((w.B, w.Hkv, w.T, w.d))
    V64 = np.empty_like(K64)
    L64 = np.empty((w.B, w.Hkv, w.nL, w.d))
    rawdt = np.float32 if w.dtype == "f32" else np.uint16
    Qr = np.empty(Q64.shape, rawdt)
    Kr = np.empty(K64.shape, rawdt)
    Vr = np.empty(K64.shape, rawdt)
    Lr = np.empty(L64.shape, rawdt)
    for b in range(w.B):
        Q64[b], Qr[b] = q_rows(w, b, np.arange(w.H), np.arange(w.N))
        for g in range(w.Hkv):
            K64[b, g], Kr[b, g] = k_rows(w, b, g, 0, w.T)
            V64[b, g], Vr[b, g] = v_rows(w, b, g, 0, w.T)
            L64[b, g], Lr[b, g] = l_rows(w, b, g, 0, w.nL)
    return {"Q": (Q64, Qr), "K": (K64, Kr), "V": (V64, Vr), "L": (L64, Lr)}
