// attend_prefill.cu -- chunk attention and fusion for many queries (CUDA-core path).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Abstract
// (attend inside each retrieved chunk, fuse by retrieval scores); Sec. 3
// "Hierarchical softmax"; Sec. 4 "Architecture" (a group's heads share the
// retrieved chunks, so each chunk is gathered once per group).
//
// One CTA per query group (b, g, i), one warp per head of the group.  Each
// selected chunk's keys and values are staged once in shared memory and used
// by all G warps.  The fusion weights are known before the first chunk (they
// depend only on the slot scores), so every chunk output is folded into the
// accumulator as soon as it is normalised: no running rescale is needed.
// This path serves float32 inputs and every shape; bf16 inputs with d = 128 and
// C = 64 take the tensor-core kernel when it is available.
#include "attend_simt.cuh"

namespace hils {
namespace {

template <typename Tin, typename Tout, int D>
__global__ void attend_prefill_simt_kernel(Dims p, const Tin *__restrict__ Q, const Tin *__restrict__ K,
                                           const Tin *__restrict__ V, const int32_t *__restrict__ sel_idx,
                                           const float *__restrict__ sel_score, Tout *__restrict__ O)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Tin *Ks = reinterpret_cast<Tin *>(smem_raw);
    Tin *Vs = Ks + (size_t)p.C * D;
    float *qsm = reinterpret_cast<float *>(Vs + (size_t)p.C * D);   // [G][D]
    float *wsm = qsm + (size_t)p.G * D;                              // [G][k+1]
    int *chunk = reinterpret_cast<int *>(wsm + (size_t)p.G * (p.k + 1));  // [k+1]

    const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * p.G + warp;
    const long long pos = (long long)p.q_offset + i;
    const int ci = (int)(pos / p.C);
    const int ns = p.k + 1;

    const size_t row_h = (((size_t)b * p.H + h) * p.N) + i;
    for (int x = lane; x < D; x += 32) qsm[warp * D + x] = to_float(Q[row_h * D + x]) * p.scale;
    const int32_t *si = sel_idx + ((((size_t)b * p.Hkv + g) * p.N) + i) * p.k;
    for (int j = threadIdx.x; j < ns; j += blockDim.x) chunk[j] = (j < p.k) ? si[j] : ci;
    warp_fusion_weights(sel_score + row_h * ns, ns, 0, ns, wsm + warp * ns);

    float acc[D / 32];
#pragma unroll
    for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;

    const Tin *Kbg = K + ((size_t)b * p.Hkv + g) * p.T * D;
    const Tin *Vbg = V + ((size_t)b * p.Hkv + g) * p.T * D;
    __syncthreads();
    for (int j = 0; j < ns; ++j) {
        const int c = chunk[j];
        if (c < 0) continue;
        const int n_vis = (int)min((long long)p.C, pos - (long long)c * p.C + 1);
        __syncthreads();
        stage_rows<Tin, D>(Ks, Kbg + (size_t)c * p.C * D, n_vis);
        stage_rows<Tin, D>(Vs, Vbg + (size_t)c * p.C * D, n_vis);
        __syncthreads();
        warp_attend_chunk<Tin, D>(qsm + warp * D, Ks, Vs, n_vis, wsm[warp * ns + j], acc);
    }
#pragma unroll
    for (int x = 0; x < D / 32; ++x) store_out(O + row_h * D + lane * (D / 32) + x, acc[x]);
}

template <typename Tin, typename Tout, int D>
cudaError_t launch_t(const Dims &p, const void *Q, const void *K, const void *V, const int32_t *sel_idx,
                     const float *sel_score, void *O, cudaStream_t s)
{
    const size_t smem = 2 * (size_t)p.C * D * sizeof(Tin) + (size_t)p.G * D * sizeof(float) +
                        (size_t)p.G * (p.k + 1) * sizeof(float) + (size_t)(p.k + 1) * sizeof(int);
    auto kern = attend_prefill_simt_kernel<Tin, Tout, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.N, p.Hkv, p.B);
    kern<<<grid, 32 * p.G, smem, s>>>(p, static_cast<const Tin *>(Q), static_cast<const Tin *>(K),
                                      static_cast<const Tin *>(V), sel_idx, sel_score, static_cast<Tout *>(O));
    return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t launch_d(const Dims &p, const void *Q, const void *K, const void *V, const int32_t *sel_idx,
                     const float *sel_score, void *O, cudaStream_t s)
{
    return p.d == 64 ? launch_t<Tin, Tout, 64>(p, Q, K, V, sel_idx, sel_score, O, s)
                     : launch_t<Tin, Tout, 128>(p, Q, K, V, sel_idx, sel_score, O, s);
}

}  // namespace

cudaError_t launch_attend_prefill_simt(const Dims &p, hils_dtype in, hils_dtype out, const void *Q,
                                       const void *K, const void *V, const int32_t *sel_idx,
                                       const float *sel_score, void *O, cudaStream_t s)
{
    if (in == HILS_F32)
        return out == HILS_F32 ? launch_d<float, float>(p, Q, K, V, sel_idx, sel_score, O, s)
                               : launch_d<float, __nv_bfloat16>(p, Q, K, V, sel_idx, sel_score, O, s);
    return out == HILS_F32 ? launch_d<__nv_bfloat16, float>(p, Q, K, V, sel_idx, sel_score, O, s)
                           : launch_d<__nv_bfloat16, __nv_bfloat16>(p, Q, K, V, sel_idx, sel_score, O, s);
}

}  // namespace hils
