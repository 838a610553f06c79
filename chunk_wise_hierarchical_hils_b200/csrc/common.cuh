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

}  // namespace hils
