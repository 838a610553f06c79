// warp_topk.cuh -- one warp keeps the K largest of a stream of 64-bit keys (K = 32 or 64), for the
// decode selection's top-k ("Hierarchical Sparse Attention Done Right", Sec. 3 Methodology, "Sparse
// training": keep the top-K chunks).
//
// The list is sorted descending across the warp: element e = r * 32 + lane sits in register r of lane
// `lane` (KR = K / 32 registers per lane).  Keys are distinct and non-zero; 0 marks an empty place.
// A batch of 32 new keys (one per lane) is sorted by a bitonic network of shuffles and merged: the
// elementwise maximum of the list and the reversed batch holds the K largest of both as a bitonic
// sequence, which a bitonic merge sorts.  A batch none of whose keys beats the list's last element is
// skipped after one vote.  Every lane of the warp must call these functions together.
#pragma once

#include <stdint.h>

namespace hils {
namespace wtopk {

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m)
{
    const uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, (uint32_t)(v >> 32), m);
    return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src)
{
    const uint32_t lo = __shfl_sync(0xFFFFFFFFu, (uint32_t)v, src);
    const uint32_t hi = __shfl_sync(0xFFFFFFFFu, (uint32_t)(v >> 32), src);
    return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t umax(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t umin(uint64_t a, uint64_t b) { return a < b ? a : b; }

// compare-exchange with the lane `stride` away: the lower lane keeps the larger key when the block
// runs descending
__device__ __forceinline__ uint64_t cx(uint64_t x, int stride, bool desc)
{
    const int lane = threadIdx.x & 31;
    const uint64_t y = shfl_xor_u64(x, stride);
    const bool lower = (lane & stride) == 0;
    return (lower == desc) ? umax(x, y) : umin(x, y);
}

// sort the warp's 32 keys descending (lane 0 the largest)
__device__ __forceinline__ uint64_t sort32_desc(uint64_t x)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
        const bool desc = size == 32 || (lane & size) == 0;
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) x = cx(x, stride, desc);
    }
    return x;
}

// sort a bitonic sequence of 32 (one per lane) descending
__device__ __forceinline__ uint64_t merge32_desc(uint64_t x)
{
#pragma unroll
    for (int stride = 16; stride > 0; stride >>= 1) x = cx(x, stride, true);
    return x;
}

template <int KR>
struct List {
    uint64_t v[KR];

    __device__ __forceinline__ void clear()
    {
#pragma unroll
        for (int r = 0; r < KR; ++r) v[r] = 0ull;
    }

    // the list's last (smallest) element, in every lane
    __device__ __forceinline__ uint64_t last() const { return shfl_u64(v[KR - 1], 31); }

    // merge a batch of 32 keys (one per lane, any order, 0 = none)
    __device__ __forceinline__ void add(uint64_t x)
    {
        if (!__any_sync(0xFFFFFFFFu, x > last())) return;
        x = sort32_desc(x);
        const int lane = threadIdx.x & 31;
        const uint64_t xr = shfl_u64(x, 31 - lane);   // the batch ascending
        if constexpr (KR == 1) {
            v[0] = merge32_desc(umax(v[0], xr));
        } else {
            static_assert(KR == 2, "K = 32 or 64");
            // positions 0..31 keep the list's first half; positions 32..63 take the larger of the list's
            // second half and the ascending batch: a bitonic sequence of 64, then merged
            const uint64_t c1 = umax(v[1], xr);
            const uint64_t hi = umax(v[0], c1), lo = umin(v[0], c1);
            v[0] = merge32_desc(hi);
            v[1] = merge32_desc(lo);
        }
    }

    // element e (0 <= e < 32 * KR) of the sorted list, in every lane
    __device__ __forceinline__ uint64_t at(int e) const
    {
        uint64_t r = v[0];
        if constexpr (KR == 2)
            if (e >= 32) r = v[1];
        return shfl_u64(r, e & 31);
    }
};

// A list fed one key per lane at a time (0 = none): keys that do not beat the list's last element are
// dropped at once (they cannot enter: the list only improves), the others wait in a per-warp buffer
// of 64 keys in shared memory and are merged 32 at a time, so that the sorting networks run about
// k ln(n / k) / 32 times for n keys instead of n / 32.
template <int KR>
struct Stream {
    List<KR> L;
    uint64_t thr;    // the list's last element (warp-uniform)
    int n;           // keys waiting in buf (warp-uniform)
    uint64_t *buf;   // this warp's 64 places

    __device__ __forceinline__ void init(uint64_t *b)
    {
        L.clear();
        thr = 0ull;
        n = 0;
        buf = b;
    }

    __device__ __forceinline__ void offer(uint64_t x)
    {
        const bool pass = x > thr;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, pass);
        if (!m) return;
        const int lane = threadIdx.x & 31;
        if (pass) buf[n + __popc(m & ((1u << lane) - 1u))] = x;
        n += __popc(m);
        if (n >= 32) {
            __syncwarp();
            const uint64_t b = buf[lane];
            const uint64_t rest = (lane + 32 < n) ? buf[lane + 32] : 0ull;
            __syncwarp();
            L.add(b);
            thr = L.last();
            n -= 32;
            if (lane < n) buf[lane] = rest;
            __syncwarp();
        }
    }

    __device__ __forceinline__ void flush()
    {
        if (n > 0) {
            __syncwarp();
            const int lane = threadIdx.x & 31;
            const uint64_t b = lane < n ? buf[lane] : 0ull;
            __syncwarp();
            L.add(b);
            thr = L.last();
            n = 0;
        }
    }
};

}  // namespace wtopk
}  // namespace hils
