// decode_fused.cu -- single-token decode in one cooperative kernel: landmark scan, top-k, slot scores,
// chunk attention and fusion (bf16 in, d = 128, C = 64, G <= 16, k <= 64).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Sec. 3 Methodology, "Sparse
// training" (score every chunk summary, keep the top-K) and "Hierarchical softmax" (softmax inside
// each chunk, chunk outputs fused by a softmax over the retrieval scores); Sec. 4, "Architecture"
// (the group's heads share the chunks); Sec. 7 Analysis, "Inference latency" (per-token decode costs
// the landmark scan plus a fixed budget of k + 1 chunks).
//
// Decode is a stream: the landmark cache of every (b, g), then the k + 1 selected chunks' keys and
// values, with little arithmetic per byte.  Each (b, g) gets S CTAs (S = 1 when there are enough
// (b, g) pairs to fill the GPU, more for a few long sequences), all resident at once (a cooperative
// launch):
//   phase 1  CTA s streams its share of the landmark rows through a ring of bulk copies (a producer
//            warp, seven consumer warps), scores them with the group's mean query (the same float32
//            steps as the two-kernel selection, so both choose the same chunks) and keeps a local
//            top-k; the last of the S CTAs (atomic ticket) merges the S lists, writes the selection
//            and the per-head slot scores, and publishes them (a release flag);
//   phase 2  the S CTAs read the selection, split its k + 1 slots among themselves, stream their
//            chunks' key and value tiles through the ring (TMA, 128-byte swizzle, no multicast), and
//            attend with one warp per chunk on mma.sync tiles (decode_tiles.cuh; warp w takes chunks
//            w, w + 5, ... from stage w, so each of its barrier waits is one phase ahead); each chunk's softmax
//            is normalised on its own and the fusion weights are known, so partial outputs add; with
//            S > 1 the last CTA of the (b, g) adds the S partials in order.
// Every wait is bounded: on expiry the CTA records HILS_ERR_TIMEOUT, waits (bounded) for its own
// copies in flight and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "decode_tiles.cuh"
#include "sm100.cuh"
#include "warp_topk.cuh"

namespace hils {
namespace {

using namespace sm100;
using dtiles::kQPitch;

constexpr int kWarps = 7;                         // consumer warps (eight warps in all: two per SM
constexpr int kThreads = 32 * (kWarps + 1);       // sub-partition, so that each may hold 255 registers)
constexpr int kD = 128, kC = 64;
constexpr int kLRows = 8 * kWarps;                // landmark rows per phase-1 stage: 8 per consumer warp
constexpr uint32_t kLStage = kLRows * kD * 2;     // 14 KB
constexpr int kNL = 11;                           // phase-1 stages
constexpr uint32_t kHalf = kC * 128;              // one 64-column half of a chunk tile
constexpr uint32_t kCStage = 4 * kHalf;           // keys then values of one chunk: 32 KB
constexpr int kNC = 5;                            // phase-2 stages = phase-2 consumer warps
constexpr uint32_t kRing = 160 * 1024;
constexpr int kKeys = 4096;                       // keys region: S x k merged keys, then the slots' rows
constexpr int kPrefetch = 12;                     // selected chunks prefetched into L2 ahead of their copies
constexpr unsigned long long kDrainNs = 2000000000ull;
static_assert(kNL * kLStage <= kRing && kNC * kCStage <= kRing, "stages fit the ring");
static_assert(kNC * 16 * kD * 4 <= kRing, "the warps' partial outputs fit the ring");
static_assert(kNC <= kWarps, "a consumer warp per phase-2 stage");
static_assert((HILS_MAX_K + 1) * kD * 2 <= kKeys * 8 && 32 * HILS_MAX_K <= kKeys, "the keys region holds both uses");

struct Layout {
    uint32_t ring, keys, qs, qbar, wsm, slot_c, top, wl, cbuf, bars, misc, total;
};

__host__ __device__ inline Layout make_layout()
{
    Layout L;
    L.ring = 0;
    L.keys = kRing;
    L.qs = L.keys + kKeys * 8;
    L.qbar = L.qs + 16 * kQPitch;
    L.wsm = L.qbar + kD * 4;
    L.slot_c = L.wsm + HILS_MAX_GROUP * (HILS_MAX_K + 1) * 4;
    L.top = (L.slot_c + (HILS_MAX_K + 1) * 4 + 7) & ~7u;
    L.wl = L.top + HILS_MAX_K * 8;
    L.cbuf = L.wl + kWarps * HILS_MAX_K * 8;
    L.bars = L.cbuf + kWarps * 64 * 8;
    L.misc = L.bars + (2 * kNL + 2 * kNC) * 8;
    L.total = L.misc + 32;
    return L;
}

struct FusedArgs {
    const __nv_bfloat16 *K, *V;   // the caches (L2 prefetches of the selected chunks)
    uint64_t *cand;          // [BG][S][k] local top-k keys
    float *part;             // [BG][S][G][d] partial outputs (S > 1)
    unsigned int *tick1;     // [BG] scan tickets
    unsigned int *tick2;     // [BG] attention tickets
    unsigned int *ready;     // [BG] selection published
    int S;                   // CTAs per (b, g)
    int spl;                 // landmark rows per CTA
};

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int *p)
{
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(unsigned int *p, unsigned int v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Warp 0 merges the consumer warps' lists (wl[w][0 .. 32 KR), descending) into out[0 .. 64), descending,
// zero padded; every thread of the block calls it.
template <int KR>
__device__ __forceinline__ void merge_lists(const uint64_t *wl, uint64_t *cbuf, uint64_t *out)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (warp == 0) {
        wtopk::Stream<KR> tk;
        tk.init(cbuf);
#pragma unroll
        for (int r = 0; r < KR; ++r) tk.L.v[r] = wl[r * 32 + lane];
        tk.thr = tk.L.last();
        for (int w = 1; w < kWarps; ++w)
#pragma unroll
            for (int r = 0; r < KR; ++r) tk.offer(wl[w * 64 + r * 32 + lane]);
        tk.flush();
#pragma unroll
        for (int r = 0; r < 2; ++r) out[r * 32 + lane] = r < KR ? tk.L.v[r] : 0ull;
    }
    __syncthreads();
}

// The k largest of n keys in shared memory (each consumer warp streams a strided share, then
// merge_lists) into out[0 .. 64); every thread of the block calls it.
template <int KR>
__device__ __forceinline__ void topk_array(const uint64_t *keys, int n, uint64_t *wl, uint64_t *cbuf, uint64_t *out)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < kWarps) {
        wtopk::Stream<KR> tk;
        tk.init(cbuf + warp * 64);
        for (int e0 = warp * 32; e0 < n; e0 += kWarps * 32) tk.offer(e0 + lane < n ? keys[e0 + lane] : 0ull);
        tk.flush();
#pragma unroll
        for (int r = 0; r < KR; ++r) wl[warp * 64 + r * 32 + lane] = tk.L.v[r];
    }
    merge_lists<KR>(wl, cbuf, out);
}

// Bounded wait of one thread until *flag >= target (set by another CTA of the same (b, g), resident
// and running); false, with the abort flag set, on a device error or expiry.
__device__ __forceinline__ bool wait_flag(const unsigned int *flag, unsigned int target, unsigned long long limit_ns,
                                          volatile int *abort_flag, unsigned int *status)
{
    const long long t0 = cycle_now();
    while (ld_acquire(flag) < target) {
        if (*reinterpret_cast<volatile unsigned int *>(status) != 0u) {
            *abort_flag = 1;
            return false;
        }
        if (past_limit(t0, limit_ns)) {
            *abort_flag = 1;
            atomicExch(status, 4u /* HILS_ERR_TIMEOUT */);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

template <typename Tout, int KR>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Dims p,
                        FusedArgs a, const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ Lm,
                        int32_t *__restrict__ sel_idx, float *__restrict__ sel_score, Tout *__restrict__ O,
                        unsigned int *status, unsigned long long limit_ns)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Layout Ly = make_layout();
    uint64_t *keys = reinterpret_cast<uint64_t *>(base + Ly.keys);
    unsigned char *qs = base + Ly.qs;
    float *qbar = reinterpret_cast<float *>(base + Ly.qbar);
    float *wsm = reinterpret_cast<float *>(base + Ly.wsm);
    int *slot_c = reinterpret_cast<int *>(base + Ly.slot_c);
    uint64_t *s_top = reinterpret_cast<uint64_t *>(base + Ly.top);
    uint64_t *wl = reinterpret_cast<uint64_t *>(base + Ly.wl);
    uint64_t *cbuf = reinterpret_cast<uint64_t *>(base + Ly.cbuf);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc);
    int *s_flag = reinterpret_cast<int *>(base + Ly.misc + 4);
    int *s_nmy = reinterpret_cast<int *>(base + Ly.misc + 8);
    const uint32_t ring0 = smem_addr(base + Ly.ring), bar0 = smem_addr(base + Ly.bars);
    auto FULL1 = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    auto EMPTY1 = [&](int i) { return bar0 + 8u * (uint32_t)(kNL + i); };
    auto FULL2 = [&](int i) { return bar0 + 8u * (uint32_t)(2 * kNL + i); };
    auto EMPTY2 = [&](int i) { return bar0 + 8u * (uint32_t)(2 * kNL + kNC + i); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = a.S;
    const int bg = blockIdx.x / S, s = blockIdx.x % S, b = bg / p.Hkv, g = bg % p.Hkv;
    const int G = p.G, k = p.k, ns = k + 1;
    const long long pos = p.q_offset;   // N == 1
    const int ci = (int)(pos / kC);
    const int n_past = k > 0 ? ci : 0;
    const int c0 = min(s * a.spl, n_past), c1 = min(c0 + a.spl, n_past);
    const int n_local = c1 - c0;
    const int n_st = (n_local + kLRows - 1) / kLRows;
    const __nv_bfloat16 *Lbg = Lm + (size_t)bg * p.nL * kD;

    if (tid == 0) {
        for (int i = 0; i < kNL; ++i) {
            mbar_init(FULL1(i), 1);
            mbar_init(EMPTY1(i), kWarps);
        }
        for (int i = 0; i < kNC; ++i) {
            mbar_init(FULL2(i), 1);
            mbar_init(EMPTY2(i), 1);
        }
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    // the group's mean query scaled by scale / G (heads added in order, as the two-kernel selection
    // does) and the group's query rows, bf16, rows G..15 zero, for the attention tiles
    if (tid < kD) {
        float v[HILS_MAX_GROUP];
#pragma unroll
        for (int h = 0; h < HILS_MAX_GROUP; ++h)
            v[h] = (h < G) ? __bfloat162float(Q[((size_t)b * p.H + (size_t)g * G + h) * kD + tid]) : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < HILS_MAX_GROUP; ++h)
            if (h < G) acc += v[h];
        qbar[tid] = acc * (p.scale / (float)G);
    }
    for (int e = tid; e < 16 * 16; e += kThreads) {
        const int r = e >> 4, seg = e & 15;
        const uint4 v = (r < G) ? __ldg(reinterpret_cast<const uint4 *>(Q + ((size_t)b * p.H + (size_t)g * G + r) * kD) + seg)
                                : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(qs + r * kQPitch + seg * 16) = v;
    }
    __syncthreads();

    // ---- phase 1: landmark scan ---------------------------------------------------------------------
    bool ok = true;
    int issued1 = 0, issued2 = 0;   // copies started by the producer thread (phase 1, phase 2)
    if (warp == kWarps) {
        if (lane == 0) {
            int &issued = issued1;
            for (; issued < n_st; ++issued) {
                const int slot = issued % kNL;
                if (issued >= kNL &&
                    !mbar_wait(EMPTY1(slot), (uint32_t)(((issued / kNL) - 1) & 1), limit_ns, abort_flag, status))
                    break;
                const int r0 = c0 + issued * kLRows, nr = min(kLRows, c1 - r0);
                const uint32_t bytes = (uint32_t)nr * kD * 2;
                mbar_arrive_expect_tx(FULL1(slot), bytes);
                bulk_load(ring0 + (uint32_t)slot * kLStage, Lbg + (size_t)r0 * kD, bytes, FULL1(slot));
            }
        }
        __syncwarp();
    } else {
        // warp w scores rows 8w .. 8w + 7 of every stage: 16 lanes per landmark row, 8 elements each, four
        // rows per half warp at once (per row the same products, order and butterfly as the two-kernel
        // selection), and offers the keys to its streaming top-k list
        const int sub = lane & 15, rb = warp * 8 + (lane >> 4) * 4;
        float qv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) qv[u] = qbar[sub * 8 + u];
        wtopk::Stream<KR> tk;
        tk.init(cbuf + warp * 64);
        for (int st = 0; st < n_st; ++st) {
            const int slot = st % kNL;
            int w_ok = 1;
            if (lane == 0) w_ok = mbar_wait(FULL1(slot), (uint32_t)((st / kNL) & 1), limit_ns, abort_flag, status);
            if (!__shfl_sync(0xFFFFFFFFu, w_ok, 0)) {
                ok = false;
                break;
            }
            const int r0 = st * kLRows, nr = min(kLRows, n_local - r0);
            const __nv_bfloat16 *stg = reinterpret_cast<const __nv_bfloat16 *>(base + Ly.ring + (size_t)slot * kLStage);
            float acc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float lv[8];
                if (rb + u < nr) {
                    lds8(stg + (size_t)(rb + u) * kD + sub * 8, lv);
                } else {
#pragma unroll
                    for (int x = 0; x < 8; ++x) lv[x] = 0.f;
                }
                float a0 = 0.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) a0 = fmaf(qv[x], lv[x], a0);
                acc[u] = a0;
            }
            // the rows' sums over the half warp's 16 lanes: per row the pairwise additions of a butterfly
            // over lane distances 8, 4, 2, 1 (float addition commutes, so every lane that forms a pair
            // gets the same value), with the rows spread over the lanes as the distance halves: 4
            // shuffles instead of 16; lane bits 3 and 2 then name the row the lane holds
            const bool b3 = (lane & 8) != 0, b2 = (lane & 4) != 0;
            const float v0 = (b3 ? acc[2] : acc[0]) + __shfl_xor_sync(0xFFFFFFFFu, b3 ? acc[0] : acc[2], 8);
            const float v1 = (b3 ? acc[3] : acc[1]) + __shfl_xor_sync(0xFFFFFFFFu, b3 ? acc[1] : acc[3], 8);
            float rs = (b2 ? v1 : v0) + __shfl_xor_sync(0xFFFFFFFFu, b2 ? v0 : v1, 4);
            rs += __shfl_xor_sync(0xFFFFFFFFu, rs, 2);
            rs += __shfl_xor_sync(0xFFFFFFFFu, rs, 1);
            __syncwarp();
            if (lane == 0) mbar_arrive(EMPTY1(slot));
            // lane 4u' of each half warp (u' = 2 b3 + b2) offers row rb + u'
            const int u = (b3 ? 2 : 0) + (b2 ? 1 : 0);
            tk.offer(((lane & 3) == 0 && rb + u < nr) ? make_key(rs, c0 + r0 + rb + u) : 0ull);
        }
        if (ok) {
            tk.flush();
#pragma unroll
            for (int r = 0; r < KR; ++r) wl[warp * 64 + r * 32 + lane] = tk.L.v[r];
        }
        if (!ok) *abort_flag = 1;
    }
    __syncthreads();
    if (*abort_flag) {
        // the copies the producer started must land before the CTA exits
        if (warp == kWarps && lane == 0)
            for (int u = max(0, issued1 - kNL); u < issued1; ++u)
                mbar_drain(FULL1(u % kNL), (uint32_t)((u / kNL) & 1), kDrainNs);
        return;
    }

    // local top-k (the warps' lists merged), then the merge by the last CTA of the (b, g)
    merge_lists<KR>(wl, cbuf, s_top);
    bool merger = true;
    if (S > 1) {
        uint64_t *mine = a.cand + ((size_t)bg * S + s) * k;
        for (int j = tid; j < k; j += kThreads) mine[j] = (j < n_local) ? s_top[j] : 0ull;
        __threadfence();
        __syncthreads();
        if (tid == 0) *s_flag = (atomicAdd(&a.tick1[bg], 1u) == (unsigned)(S - 1));
        __syncthreads();
        merger = *s_flag != 0;
        if (merger) {
            __threadfence();
            const uint64_t *all = a.cand + (size_t)bg * S * k;
            for (int e = tid; e < S * k; e += kThreads) keys[e] = __ldcg(all + e);
            __syncthreads();
            topk_array<KR>(keys, S * k, wl, cbuf, s_top);
        }
    }
    unsigned char *lrows = base + Ly.keys;   // [ns][16 pieces], bf16: the slots' landmark rows
    if (merger) {
        // the selection is written and published (other CTAs of the (b, g) start their chunk copies),
        // then the slots' landmark rows are staged for the slot scores before this CTA's own chunk copies
        // start (behind them these loads would wait for the copies' bytes)
        for (int j = tid; j < k; j += kThreads) sel_idx[(size_t)bg * k + j] = key_index(s_top[j]);
        if (S > 1) {
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release(&a.ready[bg], 1u);
        }
        uint4 lv[5];
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const int e = tid + i * kThreads;
            if (e < ns * 16) {
                const int j = e >> 4, seg = e & 15;
                const int c = (j < k) ? key_index(s_top[j]) : ci;
                lv[i] = __ldg(reinterpret_cast<const uint4 *>(Lbg + (size_t)(c >= 0 ? c : 0) * kD) + seg);
            }
        }
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            const int e = tid + i * kThreads;
            if (e < ns * 16) *reinterpret_cast<uint4 *>(lrows + (size_t)e * 16) = lv[i];
        }
    } else if (tid == 0) {
        wait_flag(&a.ready[bg], 1u, limit_ns, abort_flag, status);   // the selection of this (b, g)
    }
    __syncthreads();
    if (*abort_flag) return;

    // ---- phase 2: this CTA's slots (j = s, s + S, ...) ------------------------------------------------
    // the selection is known: the producer starts the chunk copies at once, while the consumer warps
    // work out the fusion weights (the merging CTA first computes and publishes the slot scores)
    if (tid == 0) {
        int n = 0;
        for (int j = s; j < ns; j += S) {
            const int c = (j < k) ? (merger ? key_index(s_top[j]) : __ldcg(sel_idx + (size_t)bg * k + j)) : ci;
            if (c >= 0) slot_c[n++] = (c << 8) | j;
        }
        *s_nmy = n;
    }
    __syncthreads();
    const int n_my = *s_nmy;

    const int gid = lane >> 2, tig = lane & 3;
    float oacc[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[nd][e] = 0.f;
    if (warp == kWarps) {
        if (lane == 0) {
            // the chunks are scattered over a cache of many GB: their first touch is slow (address
            // translation and DRAM latency), so each one's rows are prefetched into L2 well before its
            // tile copy, keeping many chunks in flight per SM without shared memory for them
            auto prefetch = [&](int u) {
                const int c = slot_c[u] >> 8;
                const int rows = (int)min((long long)kC, (long long)p.T - (long long)c * kC);
                const size_t off = ((size_t)bg * p.T + (size_t)c * kC) * kD;
                const uint32_t bytes = (uint32_t)rows * kD * 2;
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.K + off), "r"(bytes) : "memory");
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.V + off), "r"(bytes) : "memory");
            };
            for (int u = 0; u < min(kPrefetch, n_my); ++u) prefetch(u);
            int &issued = issued2;
            for (; issued < n_my; ++issued) {
                if (issued + kPrefetch < n_my) prefetch(issued + kPrefetch);
                const int slot = issued % kNC;
                if (issued >= kNC &&
                    !mbar_wait(EMPTY2(slot), (uint32_t)(((issued / kNC) - 1) & 1), limit_ns, abort_flag, status))
                    break;
                const int row = bg * p.T + (slot_c[issued] >> 8) * kC;
                const uint32_t dst = ring0 + (uint32_t)slot * kCStage;
                mbar_arrive_expect_tx(FULL2(slot), kCStage);
                tma_load_2d(dst, &tmK, FULL2(slot), 0, row);
                tma_load_2d(dst + kHalf, &tmK, FULL2(slot), 64, row);
                tma_load_2d(dst + 2 * kHalf, &tmV, FULL2(slot), 0, row);
                tma_load_2d(dst + 3 * kHalf, &tmV, FULL2(slot), 64, row);
            }
        }
        __syncwarp();
    } else {
        constexpr int kCons = 32 * kWarps;   // consumer threads; they meet on named barrier 1
        if (merger) {
            // the per-head scores of the k slots and the own chunk, from the staged landmark rows
            for (int task = tid; task < G * ns; task += kCons) {
                const int h = task / ns, j = task % ns;
                const int c = (j < k) ? key_index(s_top[j]) : ci;
                float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
                for (int u = 0; u < 16; ++u) {
                    const int seg = (u + j) & 15;   // rotated: threads of different slots, different banks
                    float qf[8], lf[8];
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(qs + h * kQPitch + seg * 16), qf);
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(lrows + ((size_t)j * 16 + seg) * 16), lf);
#pragma unroll
                    for (int x = 0; x < 8; x += 2) {
                        a0 = fmaf(qf[x], lf[x], a0);
                        a1 = fmaf(qf[x + 1], lf[x + 1], a1);
                    }
                }
                const float r = c >= 0 ? (a0 + a1) * p.scale : -INFINITY;
                wsm[task] = r;
                sel_score[((size_t)b * p.H + (size_t)g * G + h) * ns + j] = r;
            }
            if (S > 1) __threadfence();   // other CTAs of the (b, g) read the scores
            asm volatile("bar.sync 1, %0;" ::"r"(kCons) : "memory");
            if (tid == 0 && S > 1) st_release(&a.ready[bg], 2u);
        } else {
            if (tid == 0) wait_flag(&a.ready[bg], 2u, limit_ns, abort_flag, status);   // the slot scores
            asm volatile("bar.sync 1, %0;" ::"r"(kCons) : "memory");
            if (!*abort_flag)
                for (int task = tid; task < G * ns; task += kCons)
                    wsm[task] = __ldcg(sel_score + ((size_t)b * p.H + (size_t)g * G + task / ns) * ns + task % ns);
            asm volatile("bar.sync 1, %0;" ::"r"(kCons) : "memory");
        }
        // fusion weights of every head: softmax over its slot scores
        for (int h = warp; h < G; h += kWarps) {
            float sv[3];
#pragma unroll
            for (int u = 0; u < 3; ++u) sv[u] = (lane + 32 * u < ns) ? wsm[h * ns + lane + 32 * u] : -INFINITY;
            const float mx = warp_max(fmaxf(fmaxf(sv[0], sv[1]), sv[2]));
            float z = 0.f;
#pragma unroll
            for (int u = 0; u < 3; ++u) z += (sv[u] == -INFINITY) ? 0.f : expf(sv[u] - mx);
            z = warp_sum(z);
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 3; ++u)
                if (lane + 32 * u < ns) wsm[h * ns + lane + 32 * u] = (sv[u] == -INFINITY) ? 0.f : expf(sv[u] - mx) / z;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kCons) : "memory");
        if (warp < kNC) {
            const float sl2 = p.scale * 1.4426950408889634f;
            for (int i = warp; i < n_my; i += kNC) {
                const int slot = i % kNC;
                int w_ok = 1;
                if (lane == 0) w_ok = mbar_wait(FULL2(slot), (uint32_t)((i / kNC) & 1), limit_ns, abort_flag, status);
                if (!__shfl_sync(0xFFFFFFFFu, w_ok, 0)) {
                    *abort_flag = 1;
                    break;
                }
                const int c = slot_c[i] >> 8, j = slot_c[i] & 255;
                const int n_vis = (int)min((long long)kC, pos - (long long)c * kC + 1);
                const float w0 = (gid < G) ? wsm[gid * ns + j] : 0.f;
                const float w1 = (gid + 8 < G) ? wsm[(gid + 8) * ns + j] : 0.f;
                const uint32_t kt = ring0 + (uint32_t)slot * kCStage;
                dtiles::warp_chunk_mma<kC>(smem_addr(qs), kt, kt + 2 * kHalf, n_vis, sl2, w0, w1, oacc);
                __syncwarp();
                if (lane == 0) mbar_arrive(EMPTY2(slot));
            }
        }
    }
    __syncthreads();
    if (*abort_flag) {
        if (warp == kWarps && lane == 0)
            for (int u = max(0, issued2 - kNC); u < issued2; ++u)
                mbar_drain(FULL2(u % kNC), (uint32_t)((u / kNC) & 1), kDrainNs);
        return;
    }

    // the warps' partial outputs, added in warp order, then (S > 1) the CTAs' in order
    float *wpart = reinterpret_cast<float *>(base + Ly.ring);   // [warp][16][kD]
    if (warp < kNC) {
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            const int col = nd * 8 + tig * 2;
            *reinterpret_cast<float2 *>(wpart + ((size_t)warp * 16 + gid) * kD + col) = make_float2(oacc[nd][0], oacc[nd][1]);
            *reinterpret_cast<float2 *>(wpart + ((size_t)warp * 16 + gid + 8) * kD + col) =
                make_float2(oacc[nd][2], oacc[nd][3]);
        }
    }
    __syncthreads();
    if (S == 1) {
        for (int e = tid; e < G * kD; e += kThreads) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < kNC; ++w) acc += wpart[(size_t)w * 16 * kD + e];
            store_out(O + ((size_t)b * p.H + (size_t)g * G) * kD + e, acc);
        }
        return;
    }
    float *mine = a.part + ((size_t)bg * S + s) * G * kD;
    for (int e = tid; e < G * kD; e += kThreads) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kNC; ++w) acc += wpart[(size_t)w * 16 * kD + e];
        mine[e] = acc;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) *s_flag = (atomicAdd(&a.tick2[bg], 1u) == (unsigned)(S - 1));
    __syncthreads();
    if (!*s_flag) return;
    __threadfence();
    const float *all = a.part + (size_t)bg * S * G * kD;
    for (int e = tid; e < G * kD; e += kThreads) {
        float acc = 0.f;
        for (int u = 0; u < S; ++u) acc += __ldcg(all + (size_t)u * G * kD + e);
        store_out(O + ((size_t)b * p.H + (size_t)g * G) * kD + e, acc);
    }
}

struct FusedPlan {
    int S, spl;
};

FusedPlan fused_plan(const Dims &p)
{
    static int n_sm = 0;
    if (!n_sm) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n_sm = 0;
    }
    FusedPlan f{0, 0};
    const int BG = p.B * p.Hkv;
    if (n_sm <= 0 || BG > n_sm) return f;
    const int n_past = p.k > 0 ? (int)((long long)p.q_offset / kC) : 0;
    int S = n_sm / BG;
    if (S > 32) S = 32;
    // no more CTAs than there are rows or slots to share
    const int useful = max(1, max((n_past + kLRows - 1) / kLRows, p.k + 1));
    if (S > useful) S = useful;
    f.S = S;
    f.spl = n_past > 0 ? (n_past + S - 1) / S : 0;
    return f;
}

size_t fused_ws(const Dims &p, const FusedPlan &f)
{
    const size_t BG = (size_t)p.B * p.Hkv;
    return align_up(BG * f.S * p.k * 8, 256) + align_up(BG * f.S * p.G * kD * 4, 256) + align_up(3 * BG * 4, 256);
}

}  // namespace

bool decode_fused_supported(const Dims &p, hils_dtype in)
{
    if (in != HILS_BF16 || p.d != kD || p.C != kC || p.N != 1 || p.G > 16 || p.k > HILS_MAX_K) return false;
    return fused_plan(p).S > 0;
}

size_t decode_fused_ws_bytes(const Dims &p) { return fused_ws(p, fused_plan(p)); }

cudaError_t launch_decode_fused(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                const void *L, int32_t *sel_idx, float *sel_score, void *O, void *ws,
                                const DeviceCtl &ctl, cudaStream_t s)
{
    const FusedPlan f = fused_plan(p);
    const size_t BG = (size_t)p.B * p.Hkv;
    char *w = static_cast<char *>(ws);
    FusedArgs a;
    a.K = static_cast<const __nv_bfloat16 *>(K);
    a.V = static_cast<const __nv_bfloat16 *>(V);
    a.cand = reinterpret_cast<uint64_t *>(w);
    w += align_up(BG * f.S * p.k * 8, 256);
    a.part = reinterpret_cast<float *>(w);
    w += align_up(BG * f.S * p.G * kD * 4, 256);
    a.tick1 = reinterpret_cast<unsigned int *>(w);
    a.tick2 = a.tick1 + BG;
    a.ready = a.tick2 + BG;
    a.S = f.S;
    a.spl = f.spl;
    cudaError_t e = cudaMemsetAsync(a.tick1, 0, 3 * BG * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    CUtensorMap tk, tv;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)p.B * p.Hkv * p.T};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kC};
    if (!encode_tensor_map_sw128(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, 2, dims, strides, box) ||
        !encode_tensor_map_sw128(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 2, dims, strides, box))
        return cudaErrorInvalidValue;
    const size_t smem = make_layout().total + 1024;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(BG * f.S));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(Q), *l = static_cast<const __nv_bfloat16 *>(L);
    const unsigned long long lim = (unsigned long long)ctl.wait_limit;
#define HILS_LAUNCH_FUSED(TOUT, KRV)                                                                         \
    {                                                                                                        \
        auto kern = decode_fused_kernel<TOUT, KRV>;                                                          \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);              \
        if (e != cudaSuccess) return e;                                                                      \
        e = cudaLaunchKernelEx(&cfg, kern, tk, tv, p, a, q, l, sel_idx, sel_score, static_cast<TOUT *>(O),   \
                               ctl.status, lim);                                                             \
    }
    if (out == HILS_F32) {
        if (p.k <= 32) HILS_LAUNCH_FUSED(float, 1) else HILS_LAUNCH_FUSED(float, 2)
    } else {
        if (p.k <= 32) HILS_LAUNCH_FUSED(__nv_bfloat16, 1) else HILS_LAUNCH_FUSED(__nv_bfloat16, 2)
    }
#undef HILS_LAUNCH_FUSED
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace hils
