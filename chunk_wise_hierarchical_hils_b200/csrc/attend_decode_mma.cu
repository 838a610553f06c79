// attend_decode_mma.cu -- split-K chunk attention and fusion for single-token decode on the tensor
// cores (bf16 in, d = 128, C in {64, 128}, G <= 16).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Sec. 7 Analysis (per-token
// decode touches a fixed budget of k+1 chunks); Abstract and Sec. 3 "Hierarchical softmax"
// (softmax inside each chunk, chunks fused by a softmax over the retrieval scores); Sec. 4
// "Architecture" (a GQA group's heads share the retrieved chunks).
//
// Decode moves k+1 chunks of keys and values per (b, g) and does little arithmetic on them, so the
// kernel's job is to keep the copies streaming: the arithmetic must not hold a CTA's shared memory
// longer than the copy of its next chunk takes.  The (b, g)'s k+1 chunks are split over CTAs of
// SLOTS chunks each (the split plan of the decode selection); thread 0 of a CTA starts TMA tile
// copies (128-byte swizzle, no multicast) of all its chunks at once, and one warp per chunk then
// computes, with mma.sync m16n8k16 tiles whose 16 rows are the group's G query heads (zero
// padded):
//   S = Q K_c^T   (bf16 x bf16 -> f32),
//   P = w_c * softmax(scale * S) over the visible keys, per row,
//   O_part += P V_c   (P split into a bf16 high part and a bf16 remainder, so P keeps ~16 bits),
// reading K and V with ldmatrix (transposed for V) from the swizzled tiles.  Each chunk's softmax
// is normalised on its own and the fusion weights follow from the slot scores alone, so the
// warps' partial outputs combine by plain addition: every warp writes its rows to the workspace
// and the last CTA of the (b, g) (atomic ticket) adds them in slot order.
#include <cuda.h>
#include <cuda_bf16.h>

#include "attend_simt.cuh"
#include "decode_tiles.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr unsigned long long kDrainNs = 2000000000ull;
using dtiles::kQPitch;

template <typename Tout, int C, int SLOTS>
__global__ void __launch_bounds__(32 * SLOTS, 1)
    attend_decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Dims p,
                             DecodePlan plan, const __nv_bfloat16 *__restrict__ Q, const int32_t *__restrict__ sel_idx,
                             const float *__restrict__ sel_score, float *__restrict__ partial,
                             unsigned int *__restrict__ tickets, Tout *__restrict__ O, unsigned int *status,
                             unsigned long long limit_ns)
{
    constexpr uint32_t HALF = C * 128;      // one 64-column half of a C-row tile
    constexpr uint32_t SLOT = 4 * HALF;     // K halves, then V halves
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    unsigned char *qs = base + SLOTS * SLOT;                                  // [16][kQPitch]
    float *wsm = reinterpret_cast<float *>(qs + 16 * kQPitch);               // [16][SLOTS]
    uint64_t *bars = reinterpret_cast<uint64_t *>(wsm + 16 * SLOTS);          // [SLOTS]
    __shared__ int s_chunk[SLOTS];
    __shared__ int s_last;
    __shared__ int s_abort;

    const int split = blockIdx.x, bg = blockIdx.y, b = bg / p.Hkv, g = bg % p.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;
    const long long pos = p.q_offset;   // N == 1
    const int ci = (int)(pos / C);
    const int ns = p.k + 1;
    const int j0 = split * SLOTS, j1 = min(j0 + SLOTS, ns);
    const uint32_t slot0 = smem_addr(base);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < SLOTS; ++i) mbar_init(smem_addr(&bars[i]), 1);
        fence_mbar_init();
        for (int i = 0; i < SLOTS; ++i) {
            const int j = j0 + i;
            const int c = (j >= j1) ? -1 : (j < p.k) ? sel_idx[(size_t)bg * p.k + j] : ci;
            s_chunk[i] = c;
            if (c < 0) continue;
            const int row = bg * p.T + c * C;
            const uint32_t dst = slot0 + (uint32_t)i * SLOT, bar = smem_addr(&bars[i]);
            mbar_arrive_expect_tx(bar, SLOT);
            tma_load_2d(dst, &tmK, bar, 0, row);
            tma_load_2d(dst + HALF, &tmK, bar, 64, row);
            tma_load_2d(dst + 2 * HALF, &tmV, bar, 0, row);
            tma_load_2d(dst + 3 * HALF, &tmV, bar, 64, row);
        }
    }
    // the group's query rows, bf16, rows G..15 zero (all of a thread's loads issued before its stores)
    {
        constexpr int PER = 256 / (32 * SLOTS);
        uint4 v[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = threadIdx.x + u * 32 * SLOTS, r = e >> 4, seg = e & 15;
            v[u] = (r < G) ? __ldg(reinterpret_cast<const uint4 *>(Q + ((size_t)b * p.H + (size_t)g * G + r) * kD) + seg)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = threadIdx.x + u * 32 * SLOTS, r = e >> 4, seg = e & 15;
            *reinterpret_cast<uint4 *>(qs + r * kQPitch + seg * 16) = v[u];
        }
    }
    for (int h = warp; h < G; h += SLOTS)
        warp_fusion_weights(sel_score + ((size_t)b * p.H + (size_t)g * G + h) * ns, ns, j0, j1, wsm + h * SLOTS);
    __syncthreads();

    const int gid = lane >> 2, tig = lane & 3;   // fragment row group and thread in group
    float oacc[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[nd][e] = 0.f;

    const int c = s_chunk[warp];
    bool ok = true;
    if (c >= 0) {
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait(smem_addr(&bars[warp]), 0, limit_ns, &s_abort, status) ? 1 : 0;
        ok = __shfl_sync(0xFFFFFFFFu, w_ok, 0) != 0;
    }
    if (c >= 0 && ok) {
        const uint32_t kt = slot0 + (uint32_t)warp * SLOT, vt = kt + 2 * HALF;
        const int n_vis = (int)min((long long)C, pos - (long long)c * C + 1);
        const float w0 = (gid < G) ? wsm[gid * SLOTS + warp] : 0.f;
        const float w1 = (gid + 8 < G) ? wsm[(gid + 8) * SLOTS + warp] : 0.f;
        dtiles::warp_chunk_mma<C>(smem_addr(qs), kt, vt, n_vis, p.scale * 1.4426950408889634f, w0, w1, oacc);
    }

    // every warp writes its entry (zeros for an empty slot) so that the merge can add them all
    const int n_entries = plan.nsplit2 * SLOTS;
    float *mine = partial + ((size_t)bg * n_entries + (size_t)split * SLOTS + warp) * G * kD;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
        const int col = nd * 8 + tig * 2;
        if (gid < G) *reinterpret_cast<float2 *>(mine + gid * kD + col) = make_float2(oacc[nd][0], oacc[nd][1]);
        if (gid + 8 < G)
            *reinterpret_cast<float2 *>(mine + (gid + 8) * kD + col) = make_float2(oacc[nd][2], oacc[nd][3]);
    }
    __syncthreads();
    if (threadIdx.x == 0 && s_abort) {
        // the copies must land before the CTA exits
        for (int i = 0; i < SLOTS; ++i)
            if (s_chunk[i] >= 0) mbar_drain(smem_addr(&bars[i]), 0, kDrainNs);
    }

    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&tickets[bg], 1u) == (unsigned)(plan.nsplit2 - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // each thread adds four columns over the entries in slot order, with eight entries' loads in
    // flight at a time (the entries come from L2; one at a time, the merge would be latency-bound)
    const float4 *all = reinterpret_cast<const float4 *>(partial + (size_t)bg * n_entries * G * kD);
    const int n4 = G * kD / 4;
    for (int e4 = threadIdx.x; e4 < n4; e4 += 32 * SLOTS) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int en0 = 0; en0 < n_entries; en0 += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (en0 + u < n_entries) ? __ldcg(all + (size_t)(en0 + u) * n4 + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                a.x += v[u].x;
                a.y += v[u].y;
                a.z += v[u].z;
                a.w += v[u].w;
            }
        }
        const int h = (4 * e4) / kD, x = (4 * e4) % kD;
        Tout *dst = O + ((size_t)b * p.H + (size_t)g * G + h) * kD + x;
        store_out(dst, a.x);
        store_out(dst + 1, a.y);
        store_out(dst + 2, a.z);
        store_out(dst + 3, a.w);
    }
}

template <typename Tout, int C, int SLOTS>
cudaError_t launch_cs(const Dims &p, const DecodePlan &plan, const CUtensorMap &tk, const CUtensorMap &tv,
                      const void *Q, const int32_t *sel_idx, const float *sel_score, float *partial,
                      unsigned int *tickets, void *O, const DeviceCtl &ctl, cudaStream_t s)
{
    const size_t smem = 1024 + (size_t)SLOTS * 4 * C * 128 + 16 * kQPitch + 16 * SLOTS * 4 + SLOTS * 8;
    auto kern = attend_decode_mma_kernel<Tout, C, SLOTS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.nsplit2, p.B * p.Hkv);
    kern<<<grid, 32 * SLOTS, smem, s>>>(tk, tv, p, plan, static_cast<const __nv_bfloat16 *>(Q), sel_idx, sel_score,
                                        partial, tickets, static_cast<Tout *>(O), ctl.status,
                                        (unsigned long long)ctl.wait_limit);
    return cudaGetLastError();
}

}  // namespace

bool attend_decode_mma_supported(const Dims &p, hils_dtype in)
{
    if (in != HILS_BF16 || p.d != kD || p.N != 1 || p.G > 16) return false;
    const DecodePlan plan = decode_plan(p);
    return (p.C == 64 && plan.slots_per_cta == 2) || (p.C == 128 && plan.slots_per_cta == 1);
}

cudaError_t launch_attend_decode_mma(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                     const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                     const DeviceCtl &ctl, cudaStream_t s)
{
    const DecodePlan plan = decode_plan(p);
    float *partial = static_cast<float *>(ws);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(
        static_cast<char *>(ws) +
        align_up((size_t)p.B * p.Hkv * plan.nsplit2 * plan.slots_per_cta * p.G * kD * sizeof(float), 256));
    cudaError_t e = cudaMemsetAsync(tickets, 0, (size_t)p.B * p.Hkv * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    CUtensorMap tk, tv;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)p.B * p.Hkv * p.T};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)p.C};
    if (!encode_tensor_map_sw128(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, 2, dims, strides, box) ||
        !encode_tensor_map_sw128(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 2, dims, strides, box))
        return cudaErrorInvalidValue;
    if (p.C == 64)
        return out == HILS_F32
                   ? launch_cs<float, 64, 2>(p, plan, tk, tv, Q, sel_idx, sel_score, partial, tickets, O, ctl, s)
                   : launch_cs<__nv_bfloat16, 64, 2>(p, plan, tk, tv, Q, sel_idx, sel_score, partial, tickets, O,
                                                     ctl, s);
    return out == HILS_F32
               ? launch_cs<float, 128, 1>(p, plan, tk, tv, Q, sel_idx, sel_score, partial, tickets, O, ctl, s)
               : launch_cs<__nv_bfloat16, 128, 1>(p, plan, tk, tv, Q, sel_idx, sel_score, partial, tickets, O, ctl,
                                                  s);
}

}  // namespace hils
