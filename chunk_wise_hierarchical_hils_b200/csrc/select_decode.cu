// select_decode.cu -- landmark scan and top-k for single-token decode.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Sec. 3
// "Sparse training" (score all chunk summaries, keep the top-K) and Sec. 7
// Analysis (decode cost is a fixed retrieval budget plus the landmark scan).
//
// With one query per (b, g) and up to 65,536 candidate chunks, the scan is split
// over `nsplit` CTAs per (b, g) so that the landmark cache streams through all
// SMs at HBM rate.  Each split streams its contiguous range of landmark rows
// into a ring of shared-memory stages with bulk asynchronous copies (one copy
// per stage, several stages in flight), scores them (one 16-byte piece per lane,
// a row per half warp), sorts its keys in shared memory and publishes its local
// top-k.  The last split CTA of a (b, g) (atomic ticket) merges the nsplit
// local lists -- the global top-k lies in their union -- and writes the
// selection and the per-head scores of the k slots plus the own chunk.
#include "common.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int NT = 256;          // threads per CTA
constexpr int RING = 4;          // stages in flight
constexpr int RPS = 32;          // landmark rows per stage
constexpr unsigned long long kDrainNs = 2000000000ull;

template <typename Tin, int D>
__global__ void __launch_bounds__(NT) select_decode_kernel(Dims p, DecodePlan plan, const Tin *__restrict__ Q,
                                                           const Tin *__restrict__ L, uint64_t *__restrict__ cand,
                                                           unsigned int *__restrict__ tickets,
                                                           int32_t *__restrict__ sel_idx,
                                                           float *__restrict__ sel_score, unsigned int *status,
                                                           unsigned long long limit_ns)
{
    constexpr uint32_t STAGE_BYTES = RPS * D * sizeof(Tin);
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                              // [D]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + D * sizeof(float));  // [RING]
    unsigned char *big = smem_raw + D * sizeof(float) + 128;
    unsigned char *ring = big;                                                     // [RING][STAGE_BYTES]
    uint64_t *keys = reinterpret_cast<uint64_t *>(ring + RING * STAGE_BYTES);      // [spl]
    uint64_t *mkeys = reinterpret_cast<uint64_t *>(big);                           // merge reuses the ring
    float *rows = reinterpret_cast<float *>(big);                                  // then: staged q and L rows
    __shared__ unsigned int s_hist[256];
    __shared__ unsigned long long s_ctrl[4];
    __shared__ uint64_t s_top[HILS_MAX_K];
    __shared__ int s_last;
    __shared__ int s_abort;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.y, b = bg / p.Hkv, g = bg % p.Hkv;
    const int split = blockIdx.x;
    const long long pos = p.q_offset;              // N == 1
    const int ci = (int)(pos / p.C);
    const int n_past = p.k > 0 ? ci : 0;   // k == 0: only the own chunk is used
    const int c0 = split * plan.spl;
    const int c1 = min(c0 + plan.spl, n_past);
    const int n_local = max(c1 - c0, 0);
    const int n_stages = (n_local + RPS - 1) / RPS;
    const Tin *Lbg = L + (size_t)bg * p.nL * D;
    const uint32_t bar0 = smem_addr(bars), ring0 = smem_addr(ring);

    auto issue = [&](int s) {
        const int r0 = c0 + s * RPS, nr = min(RPS, c1 - r0);
        const uint32_t bytes = (uint32_t)nr * D * sizeof(Tin);
        const uint32_t bar = bar0 + 8u * (uint32_t)(s % RING);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(ring0 + (uint32_t)(s % RING) * STAGE_BYTES, Lbg + (size_t)r0 * D, bytes, bar);
    };

    if (tid == 0) {
        for (int s = 0; s < RING; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
        s_abort = 0;
        for (int s = 0; s < min(RING, n_stages); ++s) issue(s);
    }
    if (tid < D) {
        // the G heads' values (G <= 16) loaded together, then added in head order
        float v[16];
#pragma unroll
        for (int h = 0; h < 16; ++h)
            v[h] = (h < p.G) ? to_float(Q[((size_t)b * p.H + (size_t)g * p.G + h) * D + tid]) : 0.f;
        float a = 0.f;
#pragma unroll
        for (int h = 0; h < 16; ++h)
            if (h < p.G) a += v[h];
        qs[tid] = a * (p.scale / (float)p.G);
    }
    __syncthreads();

    // ---- score this split's chunks --------------------------------------
    constexpr int LPC = D / 8;            // lanes per landmark row
    constexpr int RPW = 32 / LPC;         // rows per warp step
    const int sub = lane % LPC;
    float qv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) qv[u] = qs[sub * 8 + u];
    int s_done = 0;   // stages consumed
    for (int s = 0; s < n_stages; ++s) {
        const int slot = s % RING;
        if (!mbar_wait(bar0 + 8u * slot, (uint32_t)((s / RING) & 1), limit_ns, &s_abort, status)) s_abort = 1;
        if (!s_abort) {
            const int r0 = s * RPS, nr = min(RPS, n_local - r0);
            const Tin *st = reinterpret_cast<const Tin *>(ring + (size_t)slot * STAGE_BYTES);
            // the loop bound is warp-uniform so that every lane reaches the shuffles
            for (int rw = warp * RPW; rw < nr; rw += (NT / 32) * RPW) {
                const int rr = rw + lane / LPC;
                float lv[8];
                if (rr < nr) {
                    lds8(st + (size_t)rr * D + sub * 8, lv);
                } else {
#pragma unroll
                    for (int u = 0; u < 8; ++u) lv[u] = 0.f;
                }
                float a = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) a = fmaf(qv[u], lv[u], a);
#pragma unroll
                for (int o = LPC / 2; o; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
                if (sub == 0 && rr < nr) keys[r0 + rr] = make_key(a, c0 + r0 + rr);
            }
        }
        __syncthreads();
        if (s_abort) break;
        s_done = s + 1;
        if (tid == 0 && s + RING < n_stages) issue(s + RING);
    }
    if (tid == 0 && s_abort) {
        // after an abort: the copies of stages issued but not consumed must land before exit
        const int issued = min(n_stages, s_done + RING);
        for (int u = s_done; u < issued; ++u)
            mbar_drain(bar0 + 8u * (u % RING), (uint32_t)((u / RING) & 1), kDrainNs);
    }
    block_topk_desc(keys, n_local, min(p.k, max(n_local, 1)), s_top, s_hist, s_ctrl);

    uint64_t *mine = cand + ((size_t)bg * plan.nsplit + split) * p.k;
    for (int j = tid; j < p.k; j += NT) mine[j] = (j < n_local) ? s_top[j] : 0ull;

    // ---- last split of this (b, g) merges --------------------------------
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&tickets[bg], 1u) == (unsigned)(plan.nsplit - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int nm = plan.nsplit * p.k;
    const uint64_t *all = cand + (size_t)bg * plan.nsplit * p.k;
    for (int e = tid; e < nm; e += NT) mkeys[e] = __ldcg(all + e);
    __syncthreads();
    if (p.k > 0) block_topk_desc(mkeys, nm, p.k, s_top, s_hist, s_ctrl);

    int32_t *si = sel_idx + (size_t)bg * p.k;
    for (int j = tid; j < p.k; j += NT) si[j] = key_index(s_top[j]);

    // per-head scores of the k slots and the own chunk: stage the group's query rows and the
    // k+1 landmark rows in shared memory (all loads in flight at once), then one dot per thread
    const int ns = p.k + 1;
    float *qrows = rows;                       // [G][D]
    float *lrows = rows + (size_t)p.G * D;     // [ns][D]
    for (int e = tid; e < (p.G + ns) * (D / 8); e += NT) {
        const int rr = e / (D / 8), seg = e % (D / 8);
        const Tin *src;
        if (rr < p.G) {
            src = Q + ((size_t)b * p.H + (size_t)g * p.G + rr) * D;
        } else {
            const int j = rr - p.G;
            const int c = (j < p.k) ? key_index(s_top[j]) : ci;
            src = Lbg + (size_t)(c >= 0 ? c : 0) * D;
        }
        float v[8];
        load8(src + seg * 8, v);
        float4 *dst = reinterpret_cast<float4 *>(rows + (size_t)rr * D + seg * 8);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    __syncthreads();
    for (int task = tid; task < p.G * ns; task += NT) {
        const int h = task / ns, j = task % ns;
        const int c = (j < p.k) ? key_index(s_top[j]) : ci;
        const float *qr = qrows + (size_t)h * D, *lr = lrows + (size_t)j * D;
        float a0 = 0.f, a1 = 0.f;
        for (int x = 0; x < D; x += 2) {
            const int i0 = (x + tid) & (D - 1), i1 = (x + 1 + tid) & (D - 1);   // rotated: no bank conflicts
            a0 = fmaf(qr[i0], lr[i0], a0);
            a1 = fmaf(qr[i1], lr[i1], a1);
        }
        sel_score[((size_t)b * p.H + (size_t)g * p.G + h) * ns + j] = (c >= 0) ? (a0 + a1) * p.scale : -INFINITY;
    }
}

template <typename Tin, int D>
size_t smem_bytes(const Dims &p, const DecodePlan &plan)
{
    const size_t scan = (size_t)RING * RPS * D * sizeof(Tin) + (size_t)plan.spl * 8;
    const size_t merge = (size_t)plan.nsplit * p.k * 8;
    const size_t score = (size_t)(p.G + p.k + 1) * D * sizeof(float);
    size_t big = scan > merge ? scan : merge;
    big = big > score ? big : score;
    return D * sizeof(float) + 128 + big;
}

template <typename Tin, int D>
cudaError_t launch_t(const Dims &p, const void *Q, const void *L, int32_t *sel_idx, float *sel_score, void *ws,
                     const DeviceCtl &ctl, cudaStream_t s)
{
    const DecodePlan plan = decode_plan(p);
    uint64_t *cand = static_cast<uint64_t *>(ws);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(
        static_cast<char *>(ws) + align_up((size_t)p.B * p.Hkv * plan.nsplit * p.k * sizeof(uint64_t), 256));
    cudaError_t e = cudaMemsetAsync(tickets, 0, (size_t)p.B * p.Hkv * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    const size_t smem = smem_bytes<Tin, D>(p, plan);
    auto kern = select_decode_kernel<Tin, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.nsplit, p.B * p.Hkv);
    kern<<<grid, NT, smem, s>>>(p, plan, static_cast<const Tin *>(Q), static_cast<const Tin *>(L), cand, tickets,
                                sel_idx, sel_score, ctl.status, (unsigned long long)ctl.wait_limit);
    return cudaGetLastError();
}

}  // namespace

DecodePlan decode_plan(const Dims &p)
{
    DecodePlan plan{};
    const int n_past = p.k > 0 ? (int)((long long)p.q_offset / p.C) : 0;
    const int bg = p.B * p.Hkv;
    // aim for about four scan CTAs per SM, each with 256..4096 candidates, and a
    // merge of at most 8192 keys
    int spl = 256;
    while (spl < 4096 && (long long)bg * ((n_past + spl - 1) / spl) > 4 * 148) spl <<= 1;
    while (spl < 4096 && (long long)((n_past + spl - 1) / spl) * p.k > 8192) spl <<= 1;
    plan.spl = spl;
    plan.nsplit = n_past > 0 ? (n_past + spl - 1) / spl : 1;
    int m = 1;
    while (m < plan.nsplit * p.k) m <<= 1;
    plan.sort_n = m > spl ? m : spl;
    // attention: two selected chunks per CTA when both fit in 64 KB of shared memory
    const int ns = p.k + 1;
    const size_t chunk_bytes = 2ull * p.C * p.d * 2;   // K and V rows of one chunk, bf16
    plan.slots_per_cta = chunk_bytes <= 32768 ? 2 : 1;
    plan.nsplit2 = (ns + plan.slots_per_cta - 1) / plan.slots_per_cta;
    return plan;
}

size_t decode_select_ws_bytes(const Dims &p)
{
    const DecodePlan plan = decode_plan(p);
    return align_up((size_t)p.B * p.Hkv * plan.nsplit * p.k * sizeof(uint64_t), 256) +
           align_up((size_t)p.B * p.Hkv * sizeof(unsigned int), 256);
}

size_t decode_select_smem_bytes(const Dims &p, hils_dtype in)
{
    const DecodePlan plan = decode_plan(p);
    if (in == HILS_F32) return p.d == 64 ? smem_bytes<float, 64>(p, plan) : smem_bytes<float, 128>(p, plan);
    return p.d == 64 ? smem_bytes<__nv_bfloat16, 64>(p, plan) : smem_bytes<__nv_bfloat16, 128>(p, plan);
}

cudaError_t launch_select_decode(const Dims &p, hils_dtype in, const void *Q, const void *L, int32_t *sel_idx,
                                 float *sel_score, void *ws, const DeviceCtl &ctl, cudaStream_t s)
{
    if (in == HILS_F32)
        return p.d == 64 ? launch_t<float, 64>(p, Q, L, sel_idx, sel_score, ws, ctl, s)
                         : launch_t<float, 128>(p, Q, L, sel_idx, sel_score, ws, ctl, s);
    return p.d == 64 ? launch_t<__nv_bfloat16, 64>(p, Q, L, sel_idx, sel_score, ws, ctl, s)
                     : launch_t<__nv_bfloat16, 128>(p, Q, L, sel_idx, sel_score, ws, ctl, s);
}

}  // namespace hils
