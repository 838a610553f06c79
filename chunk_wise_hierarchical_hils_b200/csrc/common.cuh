// common.cuh -- device helpers shared by the HiLS kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "internal.h"

namespace hils {

// ---- element loads -------------------------------------------------------

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

// Eight consecutive elements starting at p (16-byte aligned for bf16,
// 32-byte run of two 16-byte loads for f32) widened to float.
__device__ __forceinline__ void load8(const float *p, float *o)
{
    float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

__device__ __forceinline__ void unpack_bf16x8(uint4 v, float *o)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = __uint_as_float(w[i] << 16);
        o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *o)
{
    unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(p)), o);
}

// Eight consecutive elements from shared memory.
__device__ __forceinline__ void lds8(const float *p, float *o)
{
    float4 a = reinterpret_cast<const float4 *>(p)[0];
    float4 b = reinterpret_cast<const float4 *>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

__device__ __forceinline__ void lds8(const __nv_bfloat16 *p, float *o)
{
    unpack_bf16x8(*reinterpret_cast<const uint4 *>(p), o);
}

__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// ---- ranking keys ----------------------------------------------------------
// A 64-bit key orders candidates exactly as the selection rule does: higher
// score first, equal scores by lower chunk index.  High word: the float's bits
// mapped to an unsigned order (-0 folded onto +0); low word: ~index.  Real keys
// are never 0, so 0 marks an empty slot.

__device__ __forceinline__ uint64_t make_key(float s, int idx)
{
    s = s + 0.0f;  // -0 -> +0: both zeros tie, as they do numerically
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

__device__ __forceinline__ int key_index(uint64_t key)
{
    return key ? static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key)) : -1;
}

// ---- warp reductions -------------------------------------------------------

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// ---- block-wide bitonic sort, descending -----------------------------------
// n is a power of two; every thread of the block must call it.
__device__ __forceinline__ void bitonic_sort_desc(uint64_t *a, int n)
{
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
                int lo = 2 * t - (t & (stride - 1));
                int hi = lo + stride;
                bool desc = ((lo & size) == 0);
                uint64_t x = a[lo], y = a[hi];
                if ((x < y) == desc) { a[lo] = y; a[hi] = x; }
            }
        }
    }
    __syncthreads();
}

// ---- block-wide top-m of 64-bit keys ---------------------------------------
// Writes the m largest of keys[0..n) to out[0..m) in descending order (out is
// padded with 0 when fewer than m keys are real).  Real keys are distinct and
// non-zero; zeros are padding.  MSB-first radix select over 8-bit digits: each
// pass histograms the keys that share the current prefix, keeps the digit at
// which the count from the top reaches the number still to take, and stops as
// soon as that digit's whole group is taken.  The m survivors are then sorted.
// Every thread of the block must call it.  hist: 256 unsigned; ctrl: 4 words.
__device__ __forceinline__ void block_topk_desc(const uint64_t *keys, int n, int m, uint64_t *out,
                                                unsigned int *hist, unsigned long long *ctrl)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    if (m <= 0) {
        __syncthreads();
        return;
    }
    int m_pow2 = 1;
    while (m_pow2 < m) m_pow2 <<= 1;
    // number of real keys
    if (tid == 0) ctrl[3] = 0ull;
    __syncthreads();
    unsigned int real = 0;
    for (int i = tid; i < n; i += nt) real += keys[i] != 0ull;
    real = (unsigned)__reduce_add_sync(0xFFFFFFFFu, real);
    if (lane == 0 && real) atomicAdd(&ctrl[3], (unsigned long long)real);
    __syncthreads();
    const int n_real = (int)ctrl[3];
    unsigned long long prefix = 0ull, mask = 0ull;
    if (n_real > m) {
        unsigned int remaining = (unsigned)m;
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += nt) hist[i] = 0u;
            __syncthreads();
            for (int i = tid; i < n; i += nt) {
                const uint64_t key = keys[i];
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns digits 255-8l .. 248-8l (highest digits first)
                unsigned int c[8], tot = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    c[e] = hist[255 - 8 * lane - e];
                    tot += c[e];
                }
                unsigned int incl = tot;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += y;
                }
                const unsigned int excl = incl - tot;   // keys in higher digits than this lane's
                const unsigned int hit = __ballot_sync(0xFFFFFFFFu, excl < remaining && incl >= remaining);
                if (lane == __ffs(hit) - 1) {
                    unsigned int above = excl;
                    int e = 0;
                    while (above + c[e] < remaining) above += c[e++];
                    const unsigned int d = 255u - 8u * lane - (unsigned)e;
                    ctrl[0] = prefix | ((unsigned long long)d << shift);
                    ctrl[1] = mask | (255ull << shift);
                    ctrl[2] = ((unsigned long long)(remaining - above) << 32) | (unsigned long long)(c[e] == remaining - above);
                }
            }
            __syncthreads();
            prefix = ctrl[0];
            mask = ctrl[1];
            remaining = (unsigned)(ctrl[2] >> 32);
            const bool done = (ctrl[2] & 1ull) != 0ull;
            __syncthreads();
            if (done) break;
        }
    }
    // collect: higher prefix, or the boundary group (all of it when the loop stopped early,
    // otherwise the single key equal to the full prefix)
    if (tid == 0) ctrl[3] = 0ull;
    for (int i = tid; i < m_pow2; i += nt) out[i] = 0ull;
    __syncthreads();
    for (int i = tid; i < n; i += nt) {
        const uint64_t key = keys[i];
        if (key != 0ull && (key & mask) >= prefix) {
            const unsigned long long slot = atomicAdd(&ctrl[3], 1ull);
            if (slot < (unsigned long long)m) out[slot] = key;
        }
    }
    if (m_pow2 > 1) bitonic_sort_desc(out, m_pow2);
    else __syncthreads();
}

}  // namespace hils
