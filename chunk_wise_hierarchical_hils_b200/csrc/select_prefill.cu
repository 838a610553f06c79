// select_prefill.cu -- landmark scoring and top-k chunk selection for many queries.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Sec. 3
// Methodology, "Sparse training": every query scores all chunk summaries and
// keeps the top-K; Sec. 4, "Architecture": under GQA the group's heads share one
// selection.  The group score of chunk c is mean_h(scale * q_h . L_c), computed
// as (scale * mean_h q_h) . L_c in float32.
//
// One thread owns one query group (b, g, i) and keeps its running top-k in a
// binary min-heap in shared memory (root = weakest kept candidate).  Heap slot e
// of thread t lives at heap[e * QT + t], so the threads of a warp always touch
// 32 distinct banks whatever their heap positions.  Landmark rows are staged
// through shared memory in tiles of LT chunks and read by all threads as
// broadcasts.  After the scan a heap sort leaves the keys in rank order.
#include "common.cuh"

namespace hils {
namespace {

constexpr int LT = 32;   // landmark rows per shared-memory tile

__device__ __forceinline__ void sift_down(uint64_t *h, int n, int stride, uint64_t x)
{
    int e = 0;
    for (;;) {
        int l = 2 * e + 1;
        if (l >= n) break;
        int r = l + 1;
        int m = (r < n && h[r * stride] < h[l * stride]) ? r : l;
        uint64_t hm = h[m * stride];
        if (hm >= x) break;
        h[e * stride] = hm;
        e = m;
    }
    h[e * stride] = x;
}

template <typename Tin, int D, int QT>
__global__ void __launch_bounds__(QT) select_prefill_kernel(Dims p, const Tin *__restrict__ Q,
                                                            const Tin *__restrict__ L,
                                                            int32_t *__restrict__ sel_idx,
                                                            float *__restrict__ sel_score)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *heap = reinterpret_cast<uint64_t *>(smem_raw);
    float *Lt = reinterpret_cast<float *>(heap + (size_t)p.k * QT);

    const int tid = threadIdx.x;
    const int g = blockIdx.y, b = blockIdx.z;
    const int i = blockIdx.x * QT + tid;
    const bool valid = i < p.N;
    const long long pos = (long long)p.q_offset + (valid ? i : 0);
    const int ci = (int)(pos / p.C);

    // scaled group-mean query
    float qs[D];
#pragma unroll
    for (int x = 0; x < D; ++x) qs[x] = 0.f;
    if (valid) {
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
    }
    const float f = p.scale / (float)p.G;
#pragma unroll
    for (int x = 0; x < D; ++x) qs[x] *= f;

    for (int e = 0; e < p.k; ++e) heap[e * QT + tid] = 0ull;

    const int last_i = min((int)(blockIdx.x + 1) * QT, p.N) - 1;
    const int c_hi = (int)(((long long)p.q_offset + last_i) / p.C);   // candidates 0 .. c_hi-1
    const Tin *Lbg = L + ((size_t)b * p.Hkv + g) * p.nL * D;

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
                const int cend = min(nt, ci - c0);
                for (int cc = 0; cc < cend; ++cc) {
                    const float4 *lr = reinterpret_cast<const float4 *>(Lt + cc * D);
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int x = 0; x < D / 4; ++x) {
                        float4 l4 = lr[x];
                        a0 = fmaf(qs[4 * x + 0], l4.x, a0);
                        a1 = fmaf(qs[4 * x + 1], l4.y, a1);
                        a2 = fmaf(qs[4 * x + 2], l4.z, a2);
                        a3 = fmaf(qs[4 * x + 3], l4.w, a3);
                    }
                    const uint64_t key = make_key((a0 + a1) + (a2 + a3), c0 + cc);
                    if (key > heap[tid]) sift_down(heap + tid, p.k, QT, key);
                }
            }
        }
    }
    if (!valid) return;

    // heap sort: repeatedly move the weakest key behind the shrinking heap,
    // leaving slots 0..k-1 in descending key order (= rank order)
    for (int n = p.k; n > 1; --n) {
        uint64_t top = heap[tid];
        uint64_t last = heap[(n - 1) * QT + tid];
        sift_down(heap + tid, n - 1, QT, last);
        heap[(n - 1) * QT + tid] = top;
    }

    const size_t row_g = (((size_t)b * p.Hkv + g) * p.N) + i;
    int32_t *si = sel_idx + row_g * p.k;
    for (int j = 0; j < p.k; ++j) si[j] = key_index(heap[j * QT + tid]);

    // per-head retrieval scores of the k slots and the own chunk
    const int ns = p.k + 1;
    for (int h = 0; h < p.G; ++h) {
        const size_t row_h = (((size_t)b * p.H + (size_t)g * p.G + h) * p.N) + i;
        const Tin *qrow = Q + row_h * D;
        float *so = sel_score + row_h * ns;
        for (int j = 0; j < ns; ++j) {
            const int c = (j < p.k) ? key_index(heap[j * QT + tid]) : ci;
            if (c < 0) { so[j] = -INFINITY; continue; }
            const Tin *lrow = Lbg + (size_t)c * D;
            float acc = 0.f;
            for (int x = 0; x < D; x += 8) {
                float qv[8], lv[8];
                load8(qrow + x, qv);
                load8(lrow + x, lv);
#pragma unroll
                for (int u = 0; u < 8; ++u) acc = fmaf(qv[u], lv[u], acc);
            }
            so[j] = acc * p.scale;
        }
    }
}

template <typename Tin, int D>
cudaError_t launch_t(const Dims &p, const void *Q, const void *L, int32_t *sel_idx, float *sel_score,
                     cudaStream_t s)
{
    constexpr int QT = 128;
    const size_t smem = (size_t)p.k * QT * sizeof(uint64_t) + (size_t)LT * D * sizeof(float);
    auto kern = select_prefill_kernel<Tin, D, QT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.N + QT - 1) / QT, p.Hkv, p.B);
    kern<<<grid, QT, smem, s>>>(p, static_cast<const Tin *>(Q), static_cast<const Tin *>(L), sel_idx,
                                sel_score);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_prefill(const Dims &p, hils_dtype in, const void *Q, const void *L,
                                  int32_t *sel_idx, float *sel_score, cudaStream_t s)
{
    if (in == HILS_F32)
        return p.d == 64 ? launch_t<float, 64>(p, Q, L, sel_idx, sel_score, s)
                         : launch_t<float, 128>(p, Q, L, sel_idx, sel_score, s);
    return p.d == 64 ? launch_t<__nv_bfloat16, 64>(p, Q, L, sel_idx, sel_score, s)
                     : launch_t<__nv_bfloat16, 128>(p, Q, L, sel_idx, sel_score, s);
}

}  // namespace hils
