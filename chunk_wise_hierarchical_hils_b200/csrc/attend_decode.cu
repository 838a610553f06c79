// attend_decode.cu -- split-K chunk attention and fusion for single-token decode.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Sec. 7
// Analysis (per-token decode touches a fixed budget of k+1 chunks, so its cost
// does not grow with the cache); Abstract and Sec. 3 "Hierarchical softmax".
//
// The k+1 selected chunks of each (b, g) are split over `nsplit2` CTAs of one
// or two chunks each.  A CTA issues bulk asynchronous copies of all its chunks'
// key and value rows at once (each chunk's rows are contiguous), so every SM
// keeps several chunks in flight, then one warp per head attends each chunk as
// it lands.  Because each chunk's softmax is normalised on its own and the
// fusion weights follow from the slot scores alone, a split's contribution is
// the plain sum of w_c * o_c over its chunks: the splits combine by addition,
// with no max or normaliser rescaling.  Each CTA writes its partial sums to the
// workspace; the last CTA of the (b, g) (atomic ticket) adds them in split order.
#include "attend_simt.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr unsigned long long kDrainNs = 2000000000ull;
constexpr int kMaxPer = 2;

template <typename Tin, typename Tout, int D>
__global__ void attend_decode_kernel(Dims p, DecodePlan plan, const Tin *__restrict__ Q,
                                     const Tin *__restrict__ K, const Tin *__restrict__ V,
                                     const int32_t *__restrict__ sel_idx, const float *__restrict__ sel_score,
                                     float *__restrict__ partial, unsigned int *__restrict__ tickets,
                                     Tout *__restrict__ O, unsigned int *status, unsigned long long limit_ns)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const size_t chunk_elems = (size_t)p.C * D;
    Tin *kv = reinterpret_cast<Tin *>(smem_raw);                                     // [per][2][C][D]
    float *qsm = reinterpret_cast<float *>(kv + 2 * chunk_elems * plan.slots_per_cta);  // [G][D]
    float *wsm = qsm + (size_t)p.G * D;                                               // [G][per]
    __shared__ uint64_t bars[kMaxPer];
    __shared__ int s_last;
    __shared__ int s_abort;
    __shared__ int s_chunk[kMaxPer];

    const int split = blockIdx.x, bg = blockIdx.y, b = bg / p.Hkv, g = bg % p.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * p.G + warp;
    const long long pos = p.q_offset;
    const int ci = (int)(pos / p.C);
    const int ns = p.k + 1;
    const int j0 = split * plan.slots_per_cta, j1 = min(j0 + plan.slots_per_cta, ns);
    const Tin *Kbg = K + (size_t)bg * p.T * D;
    const Tin *Vbg = V + (size_t)bg * p.T * D;
    const int32_t *si = sel_idx + (size_t)bg * p.k;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < j1 - j0; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
        for (int i = 0; i < j1 - j0; ++i) {
            const int j = j0 + i;
            const int c = (j < p.k) ? si[j] : ci;
            s_chunk[i] = c;
            if (c < 0) continue;
            const int n_vis = (int)min((long long)p.C, pos - (long long)c * p.C + 1);
            const uint32_t bytes = (uint32_t)n_vis * D * sizeof(Tin);
            const uint32_t bar = smem_addr(&bars[i]);
            mbar_arrive_expect_tx(bar, 2 * bytes);
            bulk_load(smem_addr(kv + 2 * chunk_elems * i), Kbg + (size_t)c * p.C * D, bytes, bar);
            bulk_load(smem_addr(kv + 2 * chunk_elems * i + chunk_elems), Vbg + (size_t)c * p.C * D, bytes, bar);
        }
    }
    const size_t row_h = (size_t)b * p.H + h;          // N == 1
    for (int x = lane; x < D; x += 32) qsm[warp * D + x] = to_float(Q[row_h * D + x]) * p.scale;
    warp_fusion_weights(sel_score + row_h * ns, ns, j0, j1, wsm + warp * plan.slots_per_cta);
    __syncthreads();

    float acc[D / 32];
#pragma unroll
    for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;
    for (int i = 0; i < j1 - j0; ++i) {
        const int c = s_chunk[i];
        if (c < 0) continue;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(smem_addr(&bars[i]), 0, limit_ns, &s_abort, status) ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
        const int n_vis = (int)min((long long)p.C, pos - (long long)c * p.C + 1);
        const Tin *Ks = kv + 2 * chunk_elems * i;
        warp_attend_chunk<Tin, D>(qsm + warp * D, Ks, Ks + chunk_elems, n_vis, wsm[warp * plan.slots_per_cta + i],
                                  acc);
    }
    __syncthreads();
    if (threadIdx.x == 0 && s_abort) {
        // the copies must land before the CTA exits
        for (int i = 0; i < j1 - j0; ++i)
            if (s_chunk[i] >= 0) mbar_drain(smem_addr(&bars[i]), 0, kDrainNs);
    }

    float *mine = partial + (((size_t)bg * plan.nsplit2 + split) * p.G + warp) * D;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) mine[lane * (D / 32) + x] = acc[x];

    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&tickets[bg], 1u) == (unsigned)(plan.nsplit2 - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const float *base = partial + ((size_t)bg * plan.nsplit2 * p.G + warp) * D;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) {
        // splits added in order, eight loads in flight at a time
        float a = 0.f;
        for (int sp0 = 0; sp0 < plan.nsplit2; sp0 += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (sp0 + u < plan.nsplit2) ? __ldcg(base + (size_t)(sp0 + u) * p.G * D + lane + 32 * x) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) a += v[u];
        }
        store_out(O + row_h * D + lane + 32 * x, a);
    }
}

template <typename Tin, typename Tout, int D>
cudaError_t launch_t(const Dims &p, const void *Q, const void *K, const void *V, const int32_t *sel_idx,
                     const float *sel_score, void *O, void *ws, const DeviceCtl &ctl, cudaStream_t s)
{
    const DecodePlan plan = decode_plan(p);
    float *partial = static_cast<float *>(ws);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(
        static_cast<char *>(ws) + align_up((size_t)p.B * p.Hkv * plan.nsplit2 * p.G * D * sizeof(float), 256));
    cudaError_t e = cudaMemsetAsync(tickets, 0, (size_t)p.B * p.Hkv * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    const size_t smem = 2 * (size_t)p.C * D * sizeof(Tin) * plan.slots_per_cta + (size_t)p.G * D * sizeof(float) +
                        (size_t)p.G * plan.slots_per_cta * sizeof(float);
    auto kern = attend_decode_kernel<Tin, Tout, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.nsplit2, p.B * p.Hkv);
    kern<<<grid, 32 * p.G, smem, s>>>(p, plan, static_cast<const Tin *>(Q), static_cast<const Tin *>(K),
                                      static_cast<const Tin *>(V), sel_idx, sel_score, partial, tickets,
                                      static_cast<Tout *>(O), ctl.status, (unsigned long long)ctl.wait_limit);
    return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t launch_d(const Dims &p, const void *Q, const void *K, const void *V, const int32_t *sel_idx,
                     const float *sel_score, void *O, void *ws, const DeviceCtl &ctl, cudaStream_t s)
{
    return p.d == 64 ? launch_t<Tin, Tout, 64>(p, Q, K, V, sel_idx, sel_score, O, ws, ctl, s)
                     : launch_t<Tin, Tout, 128>(p, Q, K, V, sel_idx, sel_score, O, ws, ctl, s);
}

}  // namespace

// Partial sums (one entry per chunk slot: the tensor-core kernel keeps one per warp, the CUDA-core
// kernel uses the first nsplit2 of them) and the (b, g) tickets.
size_t decode_attend_ws_bytes(const Dims &p)
{
    const DecodePlan plan = decode_plan(p);
    return align_up((size_t)p.B * p.Hkv * plan.nsplit2 * plan.slots_per_cta * p.G * p.d * sizeof(float), 256) +
           align_up((size_t)p.B * p.Hkv * sizeof(unsigned int), 256);
}

cudaError_t launch_attend_decode(const Dims &p, hils_dtype in, hils_dtype out, const void *Q, const void *K,
                                 const void *V, const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                 const DeviceCtl &ctl, cudaStream_t s)
{
    if (in == HILS_F32)
        return out == HILS_F32 ? launch_d<float, float>(p, Q, K, V, sel_idx, sel_score, O, ws, ctl, s)
                               : launch_d<float, __nv_bfloat16>(p, Q, K, V, sel_idx, sel_score, O, ws, ctl, s);
    return out == HILS_F32 ? launch_d<__nv_bfloat16, float>(p, Q, K, V, sel_idx, sel_score, O, ws, ctl, s)
                           : launch_d<__nv_bfloat16, __nv_bfloat16>(p, Q, K, V, sel_idx, sel_score, O, ws, ctl, s);
}

}  // namespace hils
