// landmarks.cu -- landmark generation: per chunk, a landmark query attends over the chunk's own keys.
//
// "Hierarchical Sparse Attention Done Right", Sec. 3 Methodology, "Linear surrogate for chunk mass":
// a landmark token appended to each chunk supplies a learned query; its attention over the chunk's
// keys compresses them into one key (the landmark L_c), at O(C) cost per chunk.  The same attention
// distribution gives the chunk's entropy, the bias term of the surrogate chunk mass.  For chunk c with
// key rows t (positions c*C .. min(c*C + C, T) - 1) and landmark query u_c:
//   p_t    = softmax_t(scale * <u_c, k_t>)
//   L_c    = sum_t p_t k_t
//   beta_c = -sum_t p_t ln p_t
//
// HBM-bound: every key row is read once.  One warp per chunk; each lane owns d/32 consecutive columns.
// Key rows are taken eight at a time, and the next eight rows' loads are issued before the current
// eight are used (sixteen rows in flight per lane while the warp computes); the eight logits are
// finished by butterfly sums, so every lane holds all of them, and the chunk's softmax runs online
// across the blocks of eight: running max m, running normaliser z = sum e^{s-m}, running
// y = sum e^{s-m} (s - m) for the entropy, and the lane's columns of sum e^{s-m} k.  When the max moves
// from m to m', every running sum is multiplied by e^{m-m'} and y also gains (m - m') z.  At the end
// L = acc / z and beta = ln z - y / z.
#include <cuda_bf16.h>
#include <limits.h>
#include <stdint.h>

#include "common.cuh"
#include "next_rows.h"

namespace hils {

namespace {

constexpr int kWarps = 8;     // chunks per CTA
constexpr int kRows = 8;      // key rows per online-softmax step

// E consecutive elements of row `p` owned by one lane, widened to float.
template <int E>
__device__ __forceinline__ void load_cols(const float *p, float *o)
{
    if constexpr (E == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else {
        const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
        o[0] = v.x; o[1] = v.y;
    }
}

template <int E>
__device__ __forceinline__ void load_cols(const __nv_bfloat16 *p, float *o)
{
    if constexpr (E == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
        o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xFFFF0000u);
        o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xFFFF0000u);
    } else {
        const uint32_t v = __ldg(reinterpret_cast<const unsigned int *>(p));
        o[0] = __uint_as_float(v << 16); o[1] = __uint_as_float(v & 0xFFFF0000u);
    }
}

// The raw (not yet widened) E elements of a lane, so that loads can be issued a block ahead.
template <typename Tin, int E>
struct Raw;
template <>
struct Raw<float, 4> {
    float4 v;
    __device__ __forceinline__ void load(const float *p) { v = __ldg(reinterpret_cast<const float4 *>(p)); }
    __device__ __forceinline__ void zero() { v = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void widen(float *o) const { o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w; }
};
template <>
struct Raw<float, 2> {
    float2 v;
    __device__ __forceinline__ void load(const float *p) { v = __ldg(reinterpret_cast<const float2 *>(p)); }
    __device__ __forceinline__ void zero() { v = make_float2(0.f, 0.f); }
    __device__ __forceinline__ void widen(float *o) const { o[0] = v.x; o[1] = v.y; }
};
template <>
struct Raw<__nv_bfloat16, 4> {
    uint2 v;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { v = __ldg(reinterpret_cast<const uint2 *>(p)); }
    __device__ __forceinline__ void zero() { v = make_uint2(0u, 0u); }
    __device__ __forceinline__ void widen(float *o) const
    {
        o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xFFFF0000u);
        o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xFFFF0000u);
    }
};
template <>
struct Raw<__nv_bfloat16, 2> {
    uint32_t v;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { v = __ldg(reinterpret_cast<const unsigned int *>(p)); }
    __device__ __forceinline__ void zero() { v = 0u; }
    __device__ __forceinline__ void widen(float *o) const
    {
        o[0] = __uint_as_float(v << 16); o[1] = __uint_as_float(v & 0xFFFF0000u);
    }
};

template <int E>
__device__ __forceinline__ void store_cols(float *p, const float *v)
{
    if constexpr (E == 4) *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return a | (b << 16);
}

template <int E>
__device__ __forceinline__ void store_cols(__nv_bfloat16 *p, const float *v)
{
    if constexpr (E == 4) *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    else *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(v[0], v[1]);
}

struct LandmarkArgs {
    long long units;       // (b, g, chunk) triples: B * Hkv * (c_end - c_begin)
    int span;              // c_end - c_begin
    int c_begin;
    int T, C, nL;
    float scale;
};

template <typename Tin, int D>
__global__ void __launch_bounds__(32 * kWarps, sizeof(Tin) == 2 ? 3 : 2)
landmarks_kernel(const Tin *__restrict__ K, const Tin *__restrict__ U, Tin *__restrict__ L,
                 float *__restrict__ beta, LandmarkArgs a)
{
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (unit >= a.units) return;                       // whole warps leave together; no block barrier follows
    const long long bg = unit / a.span;                // b * Hkv + g
    const int c = a.c_begin + (int)(unit - bg * a.span);
    const long long row0 = (long long)c * a.C;         // first key row of the chunk
    const int rows = (int)(a.T - row0 < (long long)a.C ? a.T - row0 : (long long)a.C);   // >= 1: c < nL

    const Tin *kc = K + ((size_t)bg * (size_t)a.T + (size_t)row0) * D + lane * E;
    const size_t lrow = ((size_t)bg * (size_t)a.nL + (size_t)c) * D + lane * E;

    float u[E];
    load_cols<E>(U + lrow, u);

    float m = -INFINITY, z = 0.f, y = 0.f;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;

    Raw<Tin, E> nxt[kRows];   // the next block's rows, loaded one block ahead
#pragma unroll
    for (int j = 0; j < kRows; ++j) {
        if (j < rows) nxt[j].load(kc + (size_t)j * D);
        else nxt[j].zero();
    }
    for (int t0 = 0; t0 < rows; t0 += kRows) {
        Raw<Tin, E> cur[kRows];   // kept raw (widened where used) to hold the registers down
        float s[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) cur[j] = nxt[j];
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
            const int t = t0 + kRows + j;
            if (t < rows) nxt[j].load(kc + (size_t)t * D);
            else nxt[j].zero();
        }
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
            float kv[E];
            cur[j].widen(kv);
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) part = fmaf(u[e], kv[e], part);
            s[j] = part;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
#pragma unroll
            for (int j = 0; j < kRows; ++j) s[j] += __shfl_xor_sync(0xFFFFFFFFu, s[j], o);
        }
        float mb = -INFINITY;
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
            s[j] = t0 + j < rows ? s[j] * a.scale : -INFINITY;
            mb = fmaxf(mb, s[j]);
        }
        const float mn = fmaxf(m, mb);                 // finite: the step holds at least one row
        if (m != -INFINITY) {                          // rescale the running sums to the new max
            const float r = expf(m - mn);
            y = r * (y + (m - mn) * z);
            z *= r;
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] *= r;
        }
        m = mn;
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
            if (t0 + j < rows) {
                const float x = s[j] - m;
                const float w = expf(x);
                z += w;
                y = fmaf(w, x, y);
                float kv[E];
                cur[j].widen(kv);
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] = fmaf(w, kv[e], acc[e]);
            }
        }
    }

    const float inv = 1.0f / z;                        // z >= 1: the max row contributes e^0
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= inv;
    store_cols<E>(L + lrow, acc);
    if (beta && lane == 0) beta[(size_t)bg * (size_t)a.nL + (size_t)c] = logf(z) - y * inv;
}

template <typename Tin, int D>
cudaError_t launch_typed(const void *K, const void *U, void *L, float *beta, const LandmarkArgs &a, cudaStream_t s)
{
    const long long blocks = (a.units + kWarps - 1) / kWarps;
    landmarks_kernel<Tin, D><<<(unsigned)blocks, 32 * kWarps, 0, s>>>(
        static_cast<const Tin *>(K), static_cast<const Tin *>(U), static_cast<Tin *>(L), beta, a);
    return cudaGetLastError();
}

}  // namespace

bool landmarks_launchable(long long B, long long Hkv, int span)
{
    const long long units = B * Hkv * (long long)span;
    return (units + kWarps - 1) / kWarps <= (long long)INT_MAX;
}

cudaError_t launch_landmarks(int B, int Hkv, int T, int d, int C, float scale, hils_dtype in, const void *K,
                             const void *U, void *L, float *beta, int c_begin, int c_end, cudaStream_t s)
{
    LandmarkArgs a;
    a.span = c_end - c_begin;
    a.units = (long long)B * Hkv * a.span;
    a.c_begin = c_begin;
    a.T = T;
    a.C = C;
    a.nL = (int)(((long long)T + C - 1) / C);
    a.scale = scale;
    if (a.units == 0) return cudaSuccess;
    if (in == HILS_BF16)
        return d == 128 ? launch_typed<__nv_bfloat16, 128>(K, U, L, beta, a, s)
                        : launch_typed<__nv_bfloat16, 64>(K, U, L, beta, a, s);
    return d == 128 ? launch_typed<float, 128>(K, U, L, beta, a, s) : launch_typed<float, 64>(K, U, L, beta, a, s);
}

}  // namespace hils
