"""Counter-based random numbers for the synthetic inputs (numpy, host side).

Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): ten rounds of two 32x32->64
multiplications mixed with xors, with a Weyl-sequence key schedule.  Being
counter-based, element ``e`` of any tensor can be produced on its own, which is
what lets the oracle rebuild exactly the slices it needs from a multi-GB input.

Normal deviates use the Box-Muller transform (Box & Muller, 1958) on two 32-bit
uniforms taken from one Philox block.  The same definition is implemented in
CUDA in ``synth/gen_cuda.cu``; a GPU test checks the two agree bit for bit.

Nothing in this module knows anything about attention.
"""
import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)

TWO_PI = 6.283185307179586  # float64 nearest to 2*pi; the CUDA side uses the same literal
INV_2_32 = 2.3283064365386963e-10  # 2**-32, exact


def philox4x32_10(ctr, key):
    """Philox4x32-10 on arrays.

    ctr: tuple of four uint64 arrays (or scalars) holding 32-bit words c0..c3.
    key: tuple of two 32-bit words k0, k1 (scalars or arrays).
    Returns four uint64 arrays holding 32-bit words.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK for c in ctr)
    k0 = np.asarray(key[0], dtype=np.uint64) & _MASK
    k1 = np.asarray(key[1], dtype=np.uint64) & _MASK
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        p0 = _M0 * c0          # < 2**64: both factors are below 2**32
        p1 = _M1 * c2
        hi0, lo0 = p0 >> _S32, p0 & _MASK
        hi1, lo1 = p1 >> _S32, p1 & _MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def _block(seed, stream, n):
    """Philox block for pair index n (uint64 array): counter (n_lo, n_hi, 0, 0), key (seed, stream)."""
    n = np.asarray(n, dtype=np.uint64)
    z = np.zeros_like(n)
    return philox4x32_10((n & _MASK, n >> _S32, z, z), (np.uint64(seed & 0xFFFFFFFF), np.uint64(stream & 0xFFFFFFFF)))


def _uniform_pair(seed, stream, n):
    x0, x1, _, _ = _block(seed, stream, n)
    u1 = (x0.astype(np.float64) + 0.5) * INV_2_32
    u2 = (x1.astype(np.float64) + 0.5) * INV_2_32
    return u1, u2


def gaussian_at(seed, stream, idx):
    """N(0,1) float64 deviates for flat element indices ``idx`` of stream ``stream``.

    Element e uses Philox block e//2; even e takes r*cos(theta), odd e r*sin(theta),
    with r = sqrt(-2 ln u1), theta = 2*pi*u2.
    """
    idx = np.asarray(idx, dtype=np.uint64)
    u1, u2 = _uniform_pair(seed, stream, idx >> np.uint64(1))
    r = np.sqrt(-2.0 * np.log(u1))
    th = TWO_PI * u2
    odd = (idx & np.uint64(1)).astype(bool)
    return np.where(odd, r * np.sin(th), r * np.cos(th))


def gaussian_range(seed, stream, start, count, block=1 << 21):
    """Deviates for the contiguous flat range [start, start+count) (float64)."""
    out = np.empty(count, dtype=np.float64)
    pos = 0
    while pos < count:
        m = min(block, count - pos)
        out[pos:pos + m] = gaussian_at(seed, stream, np.arange(start + pos, start + pos + m, dtype=np.uint64))
        pos += m
    return out


def uniform_at(seed, stream, idx):
    """U(0,1) float64 from the first word of Philox block idx: (x0 + 0.5) * 2**-32."""
    x0, _, _, _ = _block(seed, stream, idx)
    return (x0.astype(np.float64) + 0.5) * INV_2_32


def f64_to_f32(x):
    """Round to float32, nearest-even."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f32_to_bf16_bits(x32):
    """bfloat16 bit patterns (uint16) of float32 values, round-to-nearest-even (finite inputs)."""
    b = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return (r & np.uint64(0xFFFF)).astype(np.uint16)


def bf16_bits_to_f64(bits):
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)
