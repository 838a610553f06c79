// select_decode.cu -- landmark scan and top-k for single-token decode.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Sec. 3
// "Sparse training" (score all chunk summaries, keep the top-K) and Sec. 7
// Analysis (decode cost is a fixed retrieval budget plus the landmark scan).
//
// With one query per (b, g) and up to 65,536 candidate chunks, the scan is split
// over `nsplit` CTAs per (b, g) so that the landmark cache streams through all
// SMs.  Each split scores its range of chunks (half a warp, or a quarter for
// d = 64, reads one 16-byte piece per lane of each landmark row), sorts its keys
// in shared memory and publishes its local top-k to the workspace.  The last
// split CTA to finish for a (b, g) (atomic ticket) merges the nsplit local lists:
// the global top-k is contained in their union.  It then writes the selection and
// the per-head scores of the k slots plus the own chunk.
#include "common.cuh"

namespace hils {
namespace {

constexpr int NT = 256;   // threads per CTA

template <typename Tin, int D>
__global__ void __launch_bounds__(NT) select_decode_kernel(Dims p, DecodePlan plan,
                                                           const Tin *__restrict__ Q,
                                                           const Tin *__restrict__ L,
                                                           uint64_t *__restrict__ cand,
                                                           unsigned int *__restrict__ tickets,
                                                           int32_t *__restrict__ sel_idx,
                                                           float *__restrict__ sel_score)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                    // [D]
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw + D * sizeof(float));  // [sort_n]
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.y, b = bg / p.Hkv, g = bg % p.Hkv;
    const int split = blockIdx.x;
    const long long pos = p.q_offset;              // N == 1
    const int ci = (int)(pos / p.C);
    const int n_past = p.k > 0 ? ci : 0;   // k == 0: only the own chunk is used
    const int c0 = split * plan.spl;
    const int c1 = min(c0 + plan.spl, n_past);
    const Tin *Lbg = L + (size_t)bg * p.nL * D;

    if (tid < D) {
        float a = 0.f;
        for (int h = 0; h < p.G; ++h) a += to_float(Q[((size_t)b * p.H + (size_t)g * p.G + h) * D + tid]);
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
    constexpr int UNR = 4;
    const int step = (NT / 32) * RPW;
    // the loop bound is warp-uniform so that every lane reaches the shuffles
    for (int cw = c0 + warp * RPW; cw < c1; cw += step * UNR) {
        float lv[UNR][8];
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const int c = cw + lane / LPC + r * step;
            if (c < c1) {
                load8(Lbg + (size_t)c * D + sub * 8, lv[r]);
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) lv[r][u] = 0.f;
            }
        }
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            float a = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) a = fmaf(qv[u], lv[r][u], a);
#pragma unroll
            for (int o = LPC / 2; o; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
            const int c = cw + lane / LPC + r * step;
            if (sub == 0 && c < c1) keys[c - c0] = make_key(a, c);
        }
    }
    const int n_local = max(c1 - c0, 0);
    int local_n = 1;
    while (local_n < n_local) local_n <<= 1;
    for (int e = n_local + tid; e < local_n; e += NT) keys[e] = 0ull;
    if (n_local > 1) bitonic_sort_desc(keys, local_n);
    else __syncthreads();

    uint64_t *mine = cand + ((size_t)bg * plan.nsplit + split) * p.k;
    for (int j = tid; j < p.k; j += NT) mine[j] = (j < n_local) ? keys[j] : 0ull;

    // ---- last split of this (b, g) merges --------------------------------
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&tickets[bg], 1u) == (unsigned)(plan.nsplit - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int nm = plan.nsplit * p.k;
    int merge_n = 1;
    while (merge_n < nm) merge_n <<= 1;
    const uint64_t *all = cand + (size_t)bg * plan.nsplit * p.k;
    for (int e = tid; e < merge_n; e += NT) keys[e] = (e < nm) ? __ldcg(all + e) : 0ull;
    if (merge_n > 1) bitonic_sort_desc(keys, merge_n);
    else __syncthreads();

    int32_t *si = sel_idx + (size_t)bg * p.k;
    for (int j = tid; j < p.k; j += NT) si[j] = key_index(keys[j]);

    // per-head scores of the k slots and the own chunk: one warp per (head, slot)
    const int ns = p.k + 1;
    for (int task = warp; task < p.G * ns; task += NT / 32) {
        const int h = task / ns, j = task % ns;
        const int c = (j < p.k) ? key_index(keys[j]) : ci;
        float acc = 0.f;
        if (c >= 0) {
            const Tin *qrow = Q + ((size_t)b * p.H + (size_t)g * p.G + h) * D;
            const Tin *lrow = Lbg + (size_t)c * D;
            for (int x = lane; x < D; x += 32) acc = fmaf(to_float(qrow[x]), to_float(lrow[x]), acc);
            acc = warp_sum(acc);
        }
        if (lane == 0)
            sel_score[((size_t)b * p.H + (size_t)g * p.G + h) * ns + j] = (c >= 0) ? acc * p.scale : -INFINITY;
    }
}

template <typename Tin, int D>
cudaError_t launch_t(const Dims &p, const void *Q, const void *L, int32_t *sel_idx, float *sel_score,
                     void *ws, cudaStream_t s)
{
    const DecodePlan plan = decode_plan(p);
    uint64_t *cand = static_cast<uint64_t *>(ws);
    unsigned int *tickets = reinterpret_cast<unsigned int *>(
        static_cast<char *>(ws) + align_up((size_t)p.B * p.Hkv * plan.nsplit * p.k * sizeof(uint64_t), 256));
    cudaError_t e = cudaMemsetAsync(tickets, 0, (size_t)p.B * p.Hkv * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    const size_t smem = D * sizeof(float) + (size_t)plan.sort_n * sizeof(uint64_t);
    auto kern = select_decode_kernel<Tin, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(plan.nsplit, p.B * p.Hkv);
    kern<<<grid, NT, smem, s>>>(p, plan, static_cast<const Tin *>(Q), static_cast<const Tin *>(L), cand,
                                tickets, sel_idx, sel_score);
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
    // attention: one CTA per group of selected chunks, about four CTAs per SM
    const int ns = p.k + 1;
    int per = 1;
    while (per < ns && (long long)bg * ((ns + per - 1) / per) > 8 * 148) ++per;
    plan.slots_per_cta = per;
    plan.nsplit2 = (ns + per - 1) / per;
    return plan;
}

size_t decode_select_ws_bytes(const Dims &p)
{
    const DecodePlan plan = decode_plan(p);
    return align_up((size_t)p.B * p.Hkv * plan.nsplit * p.k * sizeof(uint64_t), 256) +
           align_up((size_t)p.B * p.Hkv * sizeof(unsigned int), 256);
}

cudaError_t launch_select_decode(const Dims &p, hils_dtype in, const void *Q, const void *L,
                                 int32_t *sel_idx, float *sel_score, void *ws, cudaStream_t s)
{
    if (in == HILS_F32)
        return p.d == 64 ? launch_t<float, 64>(p, Q, L, sel_idx, sel_score, ws, s)
                         : launch_t<float, 128>(p, Q, L, sel_idx, sel_score, ws, s);
    return p.d == 64 ? launch_t<__nv_bfloat16, 64>(p, Q, L, sel_idx, sel_score, ws, s)
                     : launch_t<__nv_bfloat16, 128>(p, Q, L, sel_idx, sel_score, ws, s);
}

}  // namespace hils
