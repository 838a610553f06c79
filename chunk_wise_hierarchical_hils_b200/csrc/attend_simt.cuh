// attend_simt.cuh -- one warp attends one head to one staged chunk (CUDA cores).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Abstract and
// Sec. 3 "Hierarchical softmax": the query attends inside the chunk with a
// softmax over the chunk's visible tokens only; the normalised chunk output is
// then weighted by the chunk's fusion weight.
#pragma once

#include "common.cuh"

namespace hils {

// Copy rows [0, n_rows) of a chunk (row stride D) from global to shared memory
// with 16-byte vectors, all threads of the block.
template <typename Tin, int D>
__device__ __forceinline__ void stage_rows(Tin *dst, const Tin *src, int n_rows)
{
    constexpr int VEC = 16 / sizeof(Tin);
    const int n_vec = n_rows * D / VEC;
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll 8
    for (int e = threadIdx.x; e < n_vec; e += blockDim.x) d[e] = __ldg(s + e);
}

// logit of key row krow for the scaled query in shared memory; each lane walks
// the 8-element segments in a lane-rotated order so that lanes reading
// different rows hit different banks.
template <typename Tin, int D>
__device__ __forceinline__ float dot_rotated(const float *qsm, const Tin *krow, int lane)
{
    constexpr int NSEG = D / 8;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
    for (int x = 0; x < NSEG; ++x) {
        const int seg = (x + lane) & (NSEG - 1);
        float kv[8], qv[8];
        lds8(krow + seg * 8, kv);
        lds8(qsm + seg * 8, qv);
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
            a0 = fmaf(qv[u], kv[u], a0);
            a1 = fmaf(qv[u + 1], kv[u + 1], a1);
        }
    }
    return a0 + a1;
}

// Load EPL = D/32 consecutive elements of a staged row as float (8 or 16 bytes per lane).
template <int EPL>
__device__ __forceinline__ void lds_epl(const __nv_bfloat16 *p, float *o)
{
    if constexpr (EPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        o[0] = __uint_as_float(u.x << 16); o[1] = __uint_as_float(u.x & 0xFFFF0000u);
        o[2] = __uint_as_float(u.y << 16); o[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
        o[0] = __uint_as_float(u << 16); o[1] = __uint_as_float(u & 0xFFFF0000u);
    }
}

template <int EPL>
__device__ __forceinline__ void lds_epl(const float *p, float *o)
{
    if constexpr (EPL == 4) {
        const float4 u = *reinterpret_cast<const float4 *>(p);
        o[0] = u.x; o[1] = u.y; o[2] = u.z; o[3] = u.w;
    } else {
        const float2 u = *reinterpret_cast<const float2 *>(p);
        o[0] = u.x; o[1] = u.y;
    }
}

// acc[x] (element lane * D/32 + x of the head's output) += coef * o_c, where o_c
// is the softmax-weighted mean of the staged value rows over the n_vis visible
// tokens (n_vis <= 128).
template <typename Tin, int D>
__device__ __forceinline__ void warp_attend_chunk(const float *qsm, const Tin *Ks, const Tin *Vs, int n_vis,
                                                  float coef, float *acc)
{
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    float lg[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int t = lane + 32 * m;
        lg[m] = (t < n_vis) ? dot_rotated<Tin, D>(qsm, Ks + (size_t)t * D, lane) : -INFINITY;
    }
    const float mx = warp_max(fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3])));
    float e[4], sum = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        e[m] = (lane + 32 * m < n_vis) ? expf(lg[m] - mx) : 0.f;
        sum += e[m];
    }
    sum = warp_sum(sum);
    float oc[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) oc[x] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        if (32 * m >= n_vis) break;
#pragma unroll 8
        for (int tt = 0; tt < 32; ++tt) {
            const int t = 32 * m + tt;
            const float pt = __shfl_sync(0xFFFFFFFFu, e[m], tt);
            if (t < n_vis) {
                float v[EPL];
                lds_epl<EPL>(Vs + (size_t)t * D + lane * EPL, v);
#pragma unroll
                for (int x = 0; x < EPL; ++x) oc[x] = fmaf(pt, v[x], oc[x]);
            }
        }
    }
    const float c = coef / sum;
#pragma unroll
    for (int x = 0; x < EPL; ++x) acc[x] = fmaf(c, oc[x], acc[x]);
}

// Fusion weights of the slots [j0, j1) for one head: softmax over all ns slot
// scores (-inf = empty slot).  Warp-cooperative; lane 0.. writes w[j - j0].
// The row's scores (ns <= HILS_MAX_K + 1 <= 96) are read once, all at the same time.
__device__ __forceinline__ void warp_fusion_weights(const float *score_row, int ns, int j0, int j1, float *w)
{
    const int lane = threadIdx.x & 31;
    float s[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) {
        const int j = lane + 32 * u;
        s[u] = (j < ns) ? score_row[j] : -INFINITY;
    }
    float mx = warp_max(fmaxf(fmaxf(s[0], s[1]), s[2]));
    float z = 0.f;
#pragma unroll
    for (int u = 0; u < 3; ++u) z += (s[u] == -INFINITY) ? 0.f : expf(s[u] - mx);
    z = warp_sum(z);
#pragma unroll
    for (int u = 0; u < 3; ++u) {
        const int j = lane + 32 * u;
        if (j >= j0 && j < j1) w[j - j0] = (s[u] == -INFINITY) ? 0.f : expf(s[u] - mx) / z;
    }
}

}  // namespace hils
