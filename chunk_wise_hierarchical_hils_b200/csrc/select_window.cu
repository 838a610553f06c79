// select_window.cu -- chunk selection with a local window and a per-chunk bias of the retrieval score.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1):
//   Sec. 2 Preliminary and Sec. 5 Small-scale Studies, "Experimental setup": a sliding-window branch
//   keeps the most recent tokens in every query's attention; here, chunk-aligned, the window is the
//   query's own chunk and the wc - 1 chunks before it, and retrieval ranks only the chunks before
//   the window;
//   Sec. 3 Methodology, "Linear surrogate for chunk mass": the surrogate mass of a chunk adds a
//   per-chunk bias to the query-landmark score; it enters the group score and the fusion scores.
//
// Output, in the form the chunk attention reads with k' = k + wc - 1 past slots per query:
//   sel_idx   [B][Hkv][N][k + wc - 1]: top-min(k, n_cand) candidates in rank order (higher biased
//             group score first, equal scores by lower chunk index; -1 padded to k), then the
//             window's past chunks c_i - wc + 1 .. c_i - 1 ascending (-1 below chunk 0);
//   sel_score [B][H][N][k + wc]: each slot's per-head score scale * q_h . L_c + bias_c, the own
//             chunk last (-inf for empty slots).
// n_cand = max(c_i - wc + 1, 0).  Group score = scale * mean_h q_h . L_c + bias_c in float32.
//
// Prefill (many queries): one thread per query group with its running top-k in a shared-memory
// min-heap, landmark rows staged in shared memory and read as broadcasts.  Decode (one query): one
// block per (b, g); each thread keeps a heap over a strided share of the candidates, and the block's
// radix top-k merges the heaps.
#include "common.cuh"
#include "next_rows.h"

namespace hils {
namespace {

constexpr int LT = 32;    // landmark rows per shared-memory tile (prefill)
constexpr int QT = 128;   // threads per block

__device__ __forceinline__ void heap_sift(uint64_t *h, int n, int stride, uint64_t x)
{
    int e = 0;
    for (;;) {
        const int l = 2 * e + 1;
        if (l >= n) break;
        const int r = l + 1;
        const int m = (r < n && h[r * stride] < h[l * stride]) ? r : l;
        const uint64_t hm = h[m * stride];
        if (hm >= x) break;
        h[e * stride] = hm;
        e = m;
    }
    h[e * stride] = x;
}

struct WinArgs {
    int wc;               // window chunks (>= 1)
    const float *bias;    // [B][Hkv][nL] or nullptr
};

// Scaled group-mean query of query i of (b, g): sum over the group's heads, times scale / G.
template <typename Tin, int D>
__device__ __forceinline__ void group_query(const Dims &p, const Tin *Q, int b, int g, int i, float *qs)
{
#pragma unroll
    for (int x = 0; x < D; ++x) qs[x] = 0.f;
    for (int h = 0; h < p.G; ++h) {
        const Tin *row = Q + ((((size_t)b * p.H + (size_t)g * p.G + h) * p.N) + i) * D;
#pragma unroll
        for (int x = 0; x < D; x += 8) {
            float v[8];
            load8(row + x, v);
#pragma unroll
            for (int u = 0; u < 8; ++u) qs[x + u] += v[u];
        }
    }
    const float f = p.scale / (float)p.G;
#pragma unroll
    for (int x = 0; x < D; ++x) qs[x] *= f;
}

// Chunk of slot j of a query whose top-k part is `top` (k entries, rank order): the top-k, then the
// window's past chunks ascending, then the own chunk.
__device__ __forceinline__ int slot_chunk(int j, int k, int wc, int ci, const int *top, int top_stride)
{
    if (j < k) return top[j * top_stride];
    const int c = ci - wc + 1 + (j - k);   // j = k + wc - 1 is the own chunk
    return c >= 0 ? c : -1;
}

// sel_idx row and per-head slot scores of one query group.  top[j * top_stride] = chunk of rank j.
template <typename Tin, int D>
__device__ void write_slots(const Dims &p, const WinArgs &wa, const Tin *Q, const Tin *Lbg, const float *bbg,
                            int b, int g, int i, int ci, const int *top, int top_stride, int32_t *sel_idx,
                            float *sel_score, int first, int step)
{
    const int kp = p.k + wa.wc - 1, ns = kp + 1;
    const size_t row_g = (((size_t)b * p.Hkv + g) * p.N) + i;
    for (int j = first; j < kp; j += step) sel_idx[row_g * kp + j] = slot_chunk(j, p.k, wa.wc, ci, top, top_stride);
    for (int e = first; e < p.G * ns; e += step) {
        const int h = e / ns, j = e % ns;
        const size_t row_h = (((size_t)b * p.H + (size_t)g * p.G + h) * p.N) + i;
        const int c = slot_chunk(j, p.k, wa.wc, ci, top, top_stride);
        float *so = sel_score + row_h * ns + j;
        if (c < 0) {
            *so = -INFINITY;
            continue;
        }
        const Tin *qrow = Q + row_h * D;
        const Tin *lrow = Lbg + (size_t)c * D;
        float acc = 0.f;
        for (int x = 0; x < D; x += 8) {
            float qv[8], lv[8];
            load8(qrow + x, qv);
            load8(lrow + x, lv);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = fmaf(qv[u], lv[u], acc);
        }
        *so = acc * p.scale + (bbg ? bbg[c] : 0.f);
    }
}

template <typename Tin, int D>
__global__ void __launch_bounds__(QT) select_window_prefill_kernel(Dims p, WinArgs wa, const Tin *__restrict__ Q,
                                                                   const Tin *__restrict__ L,
                                                                   int32_t *__restrict__ sel_idx,
                                                                   float *__restrict__ sel_score)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *heap = reinterpret_cast<uint64_t *>(smem_raw);
    float *Lt = reinterpret_cast<float *>(heap + (size_t)p.k * QT);
    int *top = reinterpret_cast<int *>(Lt + LT * D);   // [k][QT] chunk of each rank

    const int tid = threadIdx.x;
    const int g = blockIdx.y, b = blockIdx.z;
    const int i = blockIdx.x * QT + tid;
    const bool valid = i < p.N;
    const long long pos = (long long)p.q_offset + (valid ? i : 0);
    const int ci = (int)(pos / p.C);
    const int n_cand = max(ci - wa.wc + 1, 0);

    float qs[D];
    if (valid) group_query<Tin, D>(p, Q, b, g, i, qs);
    else
#pragma unroll
        for (int x = 0; x < D; ++x) qs[x] = 0.f;

    for (int e = 0; e < p.k; ++e) heap[e * QT + tid] = 0ull;

    const int last_i = min((int)(blockIdx.x + 1) * QT, p.N) - 1;
    const int c_hi = max((int)(((long long)p.q_offset + last_i) / p.C) - wa.wc + 1, 0);   // candidates < c_hi
    const Tin *Lbg = L + ((size_t)b * p.Hkv + g) * p.nL * D;
    const float *bbg = wa.bias ? wa.bias + ((size_t)b * p.Hkv + g) * p.nL : nullptr;

    if (p.k > 0) {
        for (int c0 = 0; c0 < c_hi; c0 += LT) {
            const int nt = min(LT, c_hi - c0);
            __syncthreads();
            for (int e = tid * 8; e < nt * D; e += QT * 8) {
                float v[8];
                load8(Lbg + (size_t)c0 * D + e, v);
                float4 *dst = reinterpret_cast<float4 *>(Lt + e);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
            __syncthreads();
            if (valid) {
                const int cend = min(nt, n_cand - c0);
                for (int cc = 0; cc < cend; ++cc) {
                    const float4 *lr = reinterpret_cast<const float4 *>(Lt + cc * D);
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int x = 0; x < D / 4; ++x) {
                        const float4 l4 = lr[x];
                        a0 = fmaf(qs[4 * x + 0], l4.x, a0);
                        a1 = fmaf(qs[4 * x + 1], l4.y, a1);
                        a2 = fmaf(qs[4 * x + 2], l4.z, a2);
                        a3 = fmaf(qs[4 * x + 3], l4.w, a3);
                    }
                    float sc = (a0 + a1) + (a2 + a3);
                    if (bbg) sc += bbg[c0 + cc];
                    const uint64_t key = make_key(sc, c0 + cc);
                    if (key > heap[tid]) heap_sift(heap + tid, p.k, QT, key);
                }
            }
        }
    }
    if (!valid) return;

    // heap sort into rank order
    for (int n = p.k; n > 1; --n) {
        const uint64_t topk = heap[tid];
        const uint64_t last = heap[(n - 1) * QT + tid];
        heap_sift(heap + tid, n - 1, QT, last);
        heap[(n - 1) * QT + tid] = topk;
    }
    for (int j = 0; j < p.k; ++j) top[j * QT + tid] = key_index(heap[j * QT + tid]);
    write_slots<Tin, D>(p, wa, Q, Lbg, bbg, b, g, i, ci, top + tid, QT, sel_idx, sel_score, 0, 1);
}

template <typename Tin, int D>
__global__ void __launch_bounds__(QT) select_window_decode_kernel(Dims p, WinArgs wa, const Tin *__restrict__ Q,
                                                                  const Tin *__restrict__ L,
                                                                  int32_t *__restrict__ sel_idx,
                                                                  float *__restrict__ sel_score, int k_pow2)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *heap = reinterpret_cast<uint64_t *>(smem_raw);        // [k][QT]
    uint64_t *out = heap + (size_t)p.k * QT;                           // [k_pow2]
    float *qsm = reinterpret_cast<float *>(out + k_pow2);              // [D]
    unsigned int *hist = reinterpret_cast<unsigned int *>(qsm + D);    // [256]
    unsigned long long *ctrl = reinterpret_cast<unsigned long long *>(hist + 256);   // [4]
    int *top = reinterpret_cast<int *>(ctrl + 4);                      // [k]

    const int tid = threadIdx.x;
    const int g = blockIdx.x, b = blockIdx.y;
    const int ci = (int)((long long)p.q_offset / p.C);
    const int n_cand = max(ci - wa.wc + 1, 0);
    const Tin *Lbg = L + ((size_t)b * p.Hkv + g) * p.nL * D;
    const float *bbg = wa.bias ? wa.bias + ((size_t)b * p.Hkv + g) * p.nL : nullptr;

    if (tid == 0) {
        float qs[D];
        group_query<Tin, D>(p, Q, b, g, 0, qs);
#pragma unroll
        for (int x = 0; x < D; ++x) qsm[x] = qs[x];
    }
    for (int e = 0; e < p.k; ++e) heap[e * QT + tid] = 0ull;
    __syncthreads();

    if (p.k > 0) {
        for (int c = tid; c < n_cand; c += QT) {
            const Tin *lrow = Lbg + (size_t)c * D;
            float a0 = 0.f, a1 = 0.f;
            for (int x = 0; x < D; x += 8) {
                float lv[8];
                load8(lrow + x, lv);
#pragma unroll
                for (int u = 0; u < 8; u += 2) {
                    a0 = fmaf(qsm[x + u], lv[u], a0);
                    a1 = fmaf(qsm[x + u + 1], lv[u + 1], a1);
                }
            }
            float sc = a0 + a1;
            if (bbg) sc += bbg[c];
            const uint64_t key = make_key(sc, c);
            if (key > heap[tid]) heap_sift(heap + tid, p.k, QT, key);
        }
    }
    __syncthreads();
    // the k best of all threads' heaps, descending (padding keys are 0)
    block_topk_desc(heap, p.k * QT, p.k, out, hist, ctrl);
    for (int j = tid; j < p.k; j += QT) top[j] = key_index(out[j]);
    __syncthreads();
    write_slots<Tin, D>(p, wa, Q, Lbg, bbg, b, g, 0, ci, top, 1, sel_idx, sel_score, tid, QT);
}

size_t decode_smem(const Dims &p, int k_pow2)
{
    return (size_t)p.k * QT * 8 + (size_t)k_pow2 * 8 + (size_t)p.d * 4 + 256 * 4 + 4 * 8 + (size_t)p.k * 4 + 16;
}

template <typename Tin, int D>
cudaError_t launch_t(const Dims &p, const WinArgs &wa, const void *Q, const void *L, int32_t *sel_idx,
                     float *sel_score, cudaStream_t s)
{
    const Tin *q = static_cast<const Tin *>(Q);
    const Tin *l = static_cast<const Tin *>(L);
    if (p.N == 1) {
        int k_pow2 = 1;
        while (k_pow2 < p.k) k_pow2 <<= 1;
        const size_t smem = decode_smem(p, k_pow2);
        auto kern = select_window_decode_kernel<Tin, D>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3(p.Hkv, p.B), QT, smem, s>>>(p, wa, q, l, sel_idx, sel_score, k_pow2);
        return cudaGetLastError();
    }
    const size_t smem = (size_t)p.k * QT * 8 + (size_t)LT * D * 4 + (size_t)p.k * QT * 4;
    auto kern = select_window_prefill_kernel<Tin, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((p.N + QT - 1) / QT, p.Hkv, p.B), QT, smem, s>>>(p, wa, q, l, sel_idx, sel_score);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_window(const Dims &p, hils_dtype in, int wc, const float *bias, const void *Q,
                                 const void *L, int32_t *sel_idx, float *sel_score, cudaStream_t s)
{
    WinArgs wa;
    wa.wc = wc;
    wa.bias = bias;
    if (in == HILS_F32)
        return p.d == 64 ? launch_t<float, 64>(p, wa, Q, L, sel_idx, sel_score, s)
                         : launch_t<float, 128>(p, wa, Q, L, sel_idx, sel_score, s);
    return p.d == 64 ? launch_t<__nv_bfloat16, 64>(p, wa, Q, L, sel_idx, sel_score, s)
                     : launch_t<__nv_bfloat16, 128>(p, wa, Q, L, sel_idx, sel_score, s);
}

}  // namespace hils
