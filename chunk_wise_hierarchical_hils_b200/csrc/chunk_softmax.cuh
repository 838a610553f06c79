// chunk_softmax.cuh -- one row of one chunk's probabilities for the tensor-core attention kernel.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Sec. 3, "Hierarchical softmax":
// inside a retrieved chunk the row's scores are normalised by a softmax over the keys the query may
// see; the chunk's result enters the output with the row's fusion weight w.  Both factors are
// applied here, so P = w * softmax(s[0 .. n_vis)) with P = 0 for masked keys.
//
// sv holds the row's 64 raw scores q.k (float bits) and is overwritten; pk receives P as 32 pairs of
// 16-bit values (key 2j in the low half): f16, or bf16 when p_bf16 is set (the caller's value tiles
// are then bf16 too).  sl2 = scale * log2(e), so exp(scale (s - m)) = 2^(sl2 s - sl2 m).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace hils {

// Pairs of scores through the f32x2 pipes; one exponential pair in POLY_PAIR_EVERY on the FMA pipe
// (exp2_poly_x2), the rest on the special-function unit.  POLY_PAIR_EVERY = 0: all on the latter.
template <int POLY_PAIR_EVERY>
__device__ __forceinline__ void chunk_softmax_row(uint32_t (&sv)[64], int n_vis, float w, float sl2,
                                                  uint32_t (&pk)[32], bool p_bf16 = false)
{
    using namespace sm100;
    if (n_vis < 64) {
#pragma unroll
        for (int j = 0; j < 64; ++j)
            if (j >= n_vis) sv[j] = __float_as_uint(-INFINITY);
    }
    float mx[8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
        mx[a] = fmax3(__uint_as_float(sv[a]), __uint_as_float(sv[8 + a]), __uint_as_float(sv[16 + a]));
#pragma unroll
    for (int j = 24; j < 64; j += 16) {
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmax3(mx[a], __uint_as_float(sv[j + a]), __uint_as_float(sv[j + 8 + a]));
    }
    const float m = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
    const uint64_t scl = f2_splat(sl2), nb = f2_splat(-m * sl2);
    uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), scl, nb);
        uint64_t e;
        if (POLY_PAIR_EVERY > 0 && j % (POLY_PAIR_EVERY > 0 ? POLY_PAIR_EVERY : 1) == POLY_PAIR_EVERY - 1) {
            e = exp2_poly_x2(x);
        } else {
            float x0, x1;
            f2_unpack(x, x0, x1);
            e = f2_pack(ex2_approx(x0), ex2_approx(x1));
        }
        ls[j & 3] = f2_add(ls[j & 3], e);
        float e0, e1;
        f2_unpack(e, e0, e1);
        sv[2 * j] = __float_as_uint(e0);
        sv[2 * j + 1] = __float_as_uint(e1);
    }
    float l0, l1;
    f2_unpack(f2_add(f2_add(ls[0], ls[1]), f2_add(ls[2], ls[3])), l0, l1);
    const uint64_t f = f2_splat(__fdividef(w, l0 + l1));
    if (p_bf16) {   // uniform over the block: one branch around the packing loop
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float a0, a1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), f), a0, a1);
            __nv_bfloat162 v2 = __floats2bfloat162_rn(a0, a1);
            pk[j] = *reinterpret_cast<uint32_t *>(&v2);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float a0, a1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), f), a0, a1);
            __half2 v2 = __floats2half2_rn(a0, a1);
            pk[j] = *reinterpret_cast<uint32_t *>(&v2);
        }
    }
}

// The same on scalar float32 pipes; one exponential in POLY_EVERY by exp2_poly (0: none).
template <int POLY_EVERY>
__device__ __forceinline__ void chunk_softmax_row_scalar(uint32_t (&sv)[64], int n_vis, float w, float sl2,
                                                         uint32_t (&pk)[32])
{
    using namespace sm100;
    if (n_vis < 64) {
#pragma unroll
        for (int j = 0; j < 64; ++j)
            if (j >= n_vis) sv[j] = __float_as_uint(-INFINITY);
    }
    float mx[8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
        mx[a] = fmax3(__uint_as_float(sv[a]), __uint_as_float(sv[8 + a]), __uint_as_float(sv[16 + a]));
#pragma unroll
    for (int j = 24; j < 64; j += 16) {
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmax3(mx[a], __uint_as_float(sv[j + a]), __uint_as_float(sv[j + 8 + a]));
    }
    const float m = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
    const float nb = -m * sl2;
    float ls[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) ls[a] = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
        const float x = fmaf(__uint_as_float(sv[j]), sl2, nb);
        const float e =
            (POLY_EVERY > 0 && j % (POLY_EVERY > 0 ? POLY_EVERY : 1) == POLY_EVERY - 1) ? exp2_poly(x) : ex2_approx(x);
        sv[j] = __float_as_uint(e);
        ls[j & 7] += e;
    }
    const float l = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
    const float f = w / l;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        __half2 v2 = __floats2half2_rn(__uint_as_float(sv[2 * j]) * f, __uint_as_float(sv[2 * j + 1]) * f);
        pk[j] = *reinterpret_cast<uint32_t *>(&v2);
    }
}

}  // namespace hils
