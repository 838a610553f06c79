// select_prefill_tc.cu -- landmark scoring and top-k chunk selection on the sm_100a tensor cores
// (bf16 in, d = 128).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Sec. 3
// Methodology, "Sparse training": every query scores all chunk summaries and
// keeps the top-K; Sec. 4, "Architecture": under GQA the group's heads share one
// selection.
//
// One CTA owns 128 rows = (128 / G) queries x the G heads of one kv-group, laid
// out query-major (row r = query * G + head) so that a query's heads sit in G
// adjacent lanes of one warp.  It streams the landmarks of chunks 0 .. c_hi in
// tiles of 64 through shared memory (TMA, 128-byte swizzle, no multicast) and
// computes every per-head score with one tcgen05.mma per tile:
//   S[row, c] = q_{query, head} . L_c      (bf16 products, f32 accumulation)
// into a double-buffered TMEM tile.  Four epilogue warps (one thread per row)
// read S, form the group score mean_h(scale * S) with a butterfly over the G
// lanes, and keep the k best (group score, chunk) keys of the row: for k <= 16
// as a sorted list in registers, updated by a branch-free insertion network
// (no memory latency on the insertion path), otherwise as a binary min-heap in
// shared memory.  With the register list, a candidate that beats the row's
// current k-th key is first queued in shared memory; the warp then inserts the
// queued keys together, so it runs the network as often as its busiest row
// needs rather than whenever any row has a candidate.  Each row carries its own head's score as the payload, so the
// per-head slot scores come out of the same pass.  Ties go to the lower chunk
// index through the key order.
#include <cuda.h>

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kD = 128;
constexpr int kTile = 64;                 // landmarks per tile
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kTmemCols = 128;       // two 64-column score buffers
constexpr unsigned long long kDrainNs = 2000000000ull;
constexpr uint32_t IDESC = idesc_bf16_f32(128, kTile, false, false);
constexpr int kQueue = 16;                // register-list path: candidates queued per row between insertions

struct Layout {
    uint32_t q, l, bar, misc, keys, pay, own, total;
};

__host__ __device__ inline Layout make_layout(int k, int nsl)
{
    Layout L;
    L.q = 0;
    L.l = 32768;
    L.bar = L.l + (uint32_t)nsl * kTileBytes;
    L.misc = L.bar + 32 * 8;
    L.keys = L.misc + 16;                                   // 8-byte aligned
    L.pay = L.keys + 8u * (uint32_t)k * kRows;
    L.own = L.pay + 4u * (uint32_t)k * kRows;
    L.total = L.own + 4u * kRows;
    return L;
}

__device__ __forceinline__ void sift_down_p(uint64_t *h, float *pl, int n, uint64_t x, float xp)
{
    int e = 0;
    for (;;) {
        const int l = 2 * e + 1;
        if (l >= n) break;
        const int r = l + 1;
        const int m = (r < n && h[r * kRows] < h[l * kRows]) ? r : l;
        const uint64_t hm = h[m * kRows];
        if (hm >= x) break;
        h[e * kRows] = hm;
        pl[e * kRows] = pl[m * kRows];
        e = m;
    }
    h[e * kRows] = x;
    pl[e * kRows] = xp;
}

// Insert key x (payload xp) into the descending list a[0..RK) if it beats the last entry: every slot
// takes its own, its upper neighbour's or the new entry's value from two comparisons, all at once.
template <int RK>
__device__ __forceinline__ void list_insert(uint64_t (&a)[RK], float (&ap)[RK], uint64_t x, float xp, bool on)
{
    bool gt[RK];
#pragma unroll
    for (int i = 0; i < RK; ++i) gt[i] = on && x > a[i];
#pragma unroll
    for (int i = RK - 1; i > 0; --i) {
        a[i] = gt[i] ? (gt[i - 1] ? a[i - 1] : x) : a[i];
        ap[i] = gt[i] ? (gt[i - 1] ? ap[i - 1] : xp) : ap[i];
    }
    a[0] = gt[0] ? x : a[0];
    ap[0] = gt[0] ? xp : ap[0];
}

// Sort a[0..RK) (RK a power of two) into descending order, payloads alongside: a bitonic
// network with every index known at compile time, so the list stays in registers.
template <int RK>
__device__ __forceinline__ void list_sort_desc(uint64_t (&a)[RK], float (&ap)[RK])
{
    static_assert(RK == 16, "the network below is written out for 16 entries");
#pragma unroll
    for (int ls = 1; ls <= 4; ++ls) {
#pragma unroll
        for (int lt = ls - 1; lt >= 0; --lt) {
            const int size = 1 << ls, stride = 1 << lt;
#pragma unroll
            for (int i = 0; i < RK; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    // blocks with (i & size) == 0 go descending, the others ascending; the last
                    // merge (size == RK) leaves everything descending
                    const bool desc = (i & size) == 0;
                    const bool swap = desc ? (a[i] < a[j]) : (a[i] > a[j]);
                    const uint64_t ki = a[i], kj = a[j];
                    const float pi = ap[i], pj = ap[j];
                    a[i] = swap ? kj : ki;
                    a[j] = swap ? ki : kj;
                    ap[i] = swap ? pj : pi;
                    ap[j] = swap ? pi : pj;
                }
            }
        }
    }
}

// The group sums of G adjacent score columns over the G lanes of a query (lane h holds head h's
// scores v[0..G) of the columns): after the rounds lane h holds the sum over the G heads of column h.
// Round r pairs lanes 2^r apart, as the butterfly sum over heads does, so each column's sum is
// associated exactly as that butterfly associates it (float addition commutes: both lanes of a pair
// form the same value); each round halves the columns a lane keeps, so G - 1 shuffles serve G columns.
template <int G>
__device__ __forceinline__ float head_sum_transposed(float (&v)[G], int h)
{
#pragma unroll
    for (int r = 0, n = G; (1 << r) < G; ++r, n >>= 1) {
        const bool bit = ((h >> r) & 1) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float keep = bit ? v[2 * i + 1] : v[2 * i];
            const float send = bit ? v[2 * i] : v[2 * i + 1];
            v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, 1 << r);
        }
    }
    return v[0];
}

__device__ __forceinline__ uint64_t shfl_xor_key(uint64_t v, int m)
{
    const uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, (uint32_t)(v >> 32), m);
    return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ void cas_desc(uint64_t &x, uint64_t &y)
{
    const uint64_t a = x, b = y;
    x = a > b ? a : b;
    y = a > b ? b : a;
}

// a bitonic sequence of 16 keys, sorted descending in place
__device__ __forceinline__ void bitonic_merge16_desc(uint64_t (&a)[16])
{
#pragma unroll
    for (int stride = 8; stride > 0; stride >>= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i & stride) == 0) cas_desc(a[i], a[i + stride]);
}

// N keys (N a power of two), sorted descending in place by a bitonic network
template <int N>
__device__ __forceinline__ void sort_desc(uint64_t (&q)[N])
{
#pragma unroll
    for (int size = 2; size <= N; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    if ((i & size) == 0 || size == N) cas_desc(q[i], q[j]);
                    else cas_desc(q[j], q[i]);
                }
            }
}

// a (descending, 16 keys) takes the 16 largest of itself and q (descending, N <= 16 keys): the tail
// of a against q reversed, elementwise maximum, is bitonic with the head of a; a merge network sorts it
template <int N>
__device__ __forceinline__ void merge_sorted(uint64_t (&a)[16], const uint64_t (&q)[N])
{
#pragma unroll
    for (int m = 0; m < N; ++m) {
        const uint64_t x = q[N - 1 - m];
        a[16 - N + m] = a[16 - N + m] > x ? a[16 - N + m] : x;
    }
    bitonic_merge16_desc(a);
}

// a (descending, 16 keys) becomes the 16 largest of a and the lane's (lane ^ m) list, descending: the
// elementwise maximum of a and the other list reversed is bitonic and holds them; a merge network sorts it
__device__ __forceinline__ void merge_with_lane(uint64_t (&a)[16], int m)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t x = shfl_xor_key(a[15 - i], m), y = shfl_xor_key(a[i], m);
        a[i] = a[i] > x ? a[i] : x;
        a[15 - i] = a[15 - i] > y ? a[15 - i] : y;
    }
    bitonic_merge16_desc(a);
}

// RES (k <= 16, G >= 2, every landmark tile of the CTA kept in TMEM): the G lanes of a query split the
// score columns (lane h ranks the columns congruent to h mod G, from the transposed head sums), merge
// their lists at the end, and read the per-head slot scores back from the resident tiles.
template <int G, int NSL, int RK, bool RES>
__global__ void __launch_bounds__(kThreads, RES ? 2 : 1)
    select_tc_kernel(const __grid_constant__ CUtensorMap tmL, Dims p, const __nv_bfloat16 *__restrict__ Q,
                     int32_t *__restrict__ sel_idx, float *__restrict__ sel_score, unsigned int *status,
                     unsigned long long limit_ns, uint32_t tmem_cols)
{
    static_assert(!RES || (RK == 16 && G >= 2), "resident tiles: register lists and two or more heads");
    constexpr int BQ = kRows / G;
    constexpr int RKN = RK > 0 ? RK : 1;   // register list length (unused when RK = 0)
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Layout Ly = make_layout(RK ? kQueue : p.k, NSL);   // register list: a kQueue-deep queue per row

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q0 = blockIdx.x * BQ, g = blockIdx.y, b = blockIdx.z;
    const int nq = min(BQ, p.N - q0);
    const int c_hi = (int)(((long long)p.q_offset + q0 + nq - 1) / p.C);   // own chunk of the last query
    const int n_tiles = c_hi / kTile + 1;

    const uint32_t sQ = smem_addr(base + Ly.q), sL = smem_addr(base + Ly.l), bar0 = smem_addr(base + Ly.bar);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 8);
    uint64_t *keys = reinterpret_cast<uint64_t *>(base + Ly.keys);
    float *pay = reinterpret_cast<float *>(base + Ly.pay);
    float *own_s = reinterpret_cast<float *>(base + Ly.own);
    auto L_FULL = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto L_EMPTY = [&](int s) { return bar0 + 8u * (uint32_t)(NSL + s); };
    auto S_FULL = [&](int s) { return bar0 + 8u * (uint32_t)(2 * NSL + s); };
    auto S_FREE = [&](int s) { return bar0 + 8u * (uint32_t)(2 * NSL + 2 + s); };
    const uint32_t MMA_DONE = bar0 + 8u * (uint32_t)(2 * NSL + 4);

    if (tid == 0) {
        for (int s = 0; s < NSL; ++s) {
            mbar_init(L_FULL(s), 1);
            mbar_init(L_EMPTY(s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(S_FULL(s), 1);
            mbar_init(S_FREE(s), 4);
        }
        mbar_init(MMA_DONE, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tensormap(&tmL);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), tmem_cols);
        tmem_relinquish();
    }
    if (RK == 0)
        for (int e = tid; e < p.k * kRows; e += kThreads) keys[e] = 0ull;
    // stage Q query-major in the 128-byte-swizzled K-major layout the MMA reads:
    // row r = query * G + head, two 64-column halves of 128 rows x 128 bytes
    // (loads issued in batches of 8 per thread before the stores: one memory latency per batch)
    for (int e0 = tid; e0 < kRows * 16; e0 += 8 * kThreads) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * kThreads;
            const int r = e >> 4, half = (e >> 3) & 1, j = e & 7;
            const int qi = r / G, h = r % G;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (e < kRows * 16 && qi < nq)
                v[u] = __ldg(reinterpret_cast<const uint4 *>(
                    Q + ((((size_t)b * p.H + (size_t)g * G + h) * p.N) + q0 + qi) * kD + half * 64 + j * 8));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u * kThreads;
            const int r = e >> 4, half = (e >> 3) & 1, j = e & 7;
            if (e < kRows * 16)
                *reinterpret_cast<uint4 *>(base + Ly.q + half * 16384u + (uint32_t)r * 128u + ((j ^ (r & 7)) << 4)) =
                    v[u];
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            const int row0 = (b * p.Hkv + g) * p.nL;
            int next = 0;
            for (int t = 0; t < n_tiles; ++t) {
                bool ok = true;
                while (next < n_tiles && (next < NSL || next <= t + NSL - 1)) {
                    const int st = next % NSL;
                    if (next >= NSL &&
                        !mbar_wait(L_EMPTY(st), (uint32_t)(((next / NSL) - 1) & 1), limit_ns, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = sL + (uint32_t)st * kTileBytes;
                    mbar_arrive_expect_tx(L_FULL(st), kTileBytes);
                    tma_load_2d(dst, &tmL, L_FULL(st), 0, row0 + next * kTile);
                    tma_load_2d(dst + kTileBytes / 2, &tmL, L_FULL(st), 64, row0 + next * kTile);
                    ++next;
                }
                if (!ok) break;
                const int st = t % NSL;
                if (!mbar_wait(L_FULL(st), (uint32_t)((t / NSL) & 1), limit_ns, abort_flag, status)) break;
                if (t >= 2 && !mbar_wait(S_FREE(t & 1), (uint32_t)(((t >> 1) - 1) & 1), limit_ns, abort_flag, status))
                    break;
                tc_fence_after();
                const uint32_t la = sL + (uint32_t)st * kTileBytes;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16_ss(tmem + (uint32_t)(RES ? t : (t & 1)) * kTile,
                                smem_desc_sw128(sQ + (s >> 2) * 16384u + (s & 3) * 32u, 16, 1024),
                                smem_desc_sw128(la + (s >> 2) * (kTileBytes / 2) + (s & 3) * 32u, 16, 1024), IDESC,
                                s > 0 ? 1u : 0u);
                mma_commit(S_FULL(t & 1));
                mma_commit(L_EMPTY(st));
            }
            mma_commit(MMA_DONE);
            mbar_drain(MMA_DONE, 0, kDrainNs);
            for (int u = max(0, next - NSL); u < next; ++u)
                mbar_drain(L_FULL(u % NSL), (uint32_t)((u / NSL) & 1), kDrainNs);
        }
        __syncwarp();
    } else if (RES && warp >= 2) {
        const int qq = warp & 3;
        const int r = 32 * qq + lane, qi = r / G, h = r % G;
        const bool valid = qi < nq;
        const long long pos = (long long)p.q_offset + q0 + qi;
        const int ci = (int)(pos / p.C);
        const float sc_g = p.scale / (float)G;
        const uint32_t trow = tmem + ((uint32_t)(32 * qq) << 16);
        uint64_t *hk = keys + r;
        uint64_t top[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) top[i] = 0ull;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            int w_ok = 1;
            if (lane == 0) w_ok = mbar_wait(S_FULL(t & 1), (uint32_t)((t >> 1) & 1), limit_ns, abort_flag, status);
            if (!__shfl_sync(0xFFFFFFFFu, w_ok, 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[32];
                tmem_ld32(trow + (uint32_t)t * kTile + 32u * half, sv);
                tmem_wait_ld();
                if (half == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(t & 1));
                }
                int qn = 0;
#pragma unroll
                for (int grp = 0; grp < 32 / G; ++grp) {
                    float v[G];
#pragma unroll
                    for (int x = 0; x < G; ++x) v[x] = __uint_as_float(sv[grp * G + x]);
                    const float gs = head_sum_transposed<G>(v, h);
                    const int c = t * kTile + 32 * half + grp * G + h;
                    const uint64_t key = make_key(gs * sc_g, c);
                    if (valid && c < ci && p.k > 0 && key > top[15]) {
                        hk[qn * kRows] = key;
                        ++qn;
                    }
                }
                // the block's queued keys (at most 32 / G <= 16) sorted by a network and merged into the
                // list
                if (__any_sync(0xFFFFFFFFu, qn > 0)) {
                    constexpr int QN = 32 / G;
                    uint64_t qk[QN];
#pragma unroll
                    for (int i = 0; i < QN; ++i) qk[i] = i < qn ? hk[i * kRows] : 0ull;
                    sort_desc<QN>(qk);
                    merge_sorted<QN>(top, qk);
                }
            }
        }
        if (__all_sync(0xFFFFFFFFu, ok)) {
            // the query's G lists into one, in every lane of the query
#pragma unroll
            for (int o = 1; o < G; o <<= 1) merge_with_lane(top, o);
            // the per-head scores of the selected chunks and of the own chunk, from the resident tiles:
            // each lane's row of a tile is staged in shared memory (the query tile's space, free once
            // the last product is done; element x of lane l at l * 64 + (x ^ l), so that neither the
            // stores nor the reads conflict) and the lane picks its columns
            float *stg = reinterpret_cast<float *>(base + Ly.q) + qq * 32 * 64;
            int cj[16];   // the selected chunks, -1 for an empty slot
            float pay[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                cj[j] = key_index(top[j]);
                pay[j] = -INFINITY;
            }
            float own = -INFINITY;
            for (int t = 0; t < n_tiles; ++t) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t sv[32];
                    tmem_ld32(trow + (uint32_t)t * kTile + 32u * half, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) stg[lane * 64 + ((32 * half + x) ^ lane)] = __uint_as_float(sv[x]);
                }
                __syncwarp();
                const int c0 = t * kTile;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int dd = cj[j] - c0;
                    if (dd >= 0 && dd < kTile) pay[j] = stg[lane * 64 + (dd ^ lane)] * p.scale;
                }
                const int dd = ci - c0;
                if (dd >= 0 && dd < kTile) own = stg[lane * 64 + (dd ^ lane)] * p.scale;
                __syncwarp();
            }
            if (valid) {
                const size_t row_g = (((size_t)b * p.Hkv + g) * p.N) + q0 + qi;
                const size_t row_h = (((size_t)b * p.H + (size_t)g * G + h) * p.N) + q0 + qi;
                const int ns = p.k + 1;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (j < p.k) {
                        if (h == 0) sel_idx[row_g * p.k + j] = cj[j];
                        sel_score[row_h * ns + j] = pay[j];   // -inf for an empty slot
                    }
                }
                sel_score[row_h * ns + p.k] = own;
            }
        }
    } else if (!RES && warp >= 2) {
        const int qq = warp & 3;
        const int r = 32 * qq + lane, qi = r / G, h = r % G;
        const bool valid = qi < nq;
        const long long pos = (long long)p.q_offset + q0 + qi;
        const int ci = (int)(pos / p.C);
        const float sc_g = p.scale / (float)G;
        const uint32_t trow = tmem + ((uint32_t)(32 * qq) << 16);
        uint64_t *hk = keys + r;
        float *hp = pay + r;
        float own = -INFINITY;
        uint64_t top[RKN];
        float topp[RKN];
#pragma unroll
        for (int i = 0; i < RKN; ++i) {
            top[i] = 0ull;
            topp[i] = 0.f;
        }
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            int w_ok = 1;
            if (lane == 0) w_ok = mbar_wait(S_FULL(t & 1), (uint32_t)((t >> 1) & 1), limit_ns, abort_flag, status);
            if (!__shfl_sync(0xFFFFFFFFu, w_ok, 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int c0 = t * kTile;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t sv[32];
                tmem_ld32(trow + (uint32_t)(t & 1) * kTile + 32u * half, sv);
                tmem_wait_ld();
                if (half == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(t & 1));
                }
                int qn = 0;   // queued candidates of this row (register-list path)
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (RK > 0 && j == kQueue) {
                        // the queue is full after kQueue candidates: insert them before going on.  The
                        // first time the list is still empty and the queue holds at most RK keys: they
                        // are copied in and sorted by a network instead of inserted one by one.
                        bool filled = false;
                        if constexpr (RKN == kQueue) {
                            if (t == 0 && half == 0) {
#pragma unroll
                                for (int i = 0; i < RKN; ++i) {
                                    const bool on = i < qn;
                                    top[i] = on ? hk[i * kRows] : 0ull;
                                    topp[i] = on ? hp[i * kRows] : 0.f;
                                }
                                list_sort_desc<RKN>(top, topp);
                                filled = true;
                            }
                        }
                        if (!filled) {
                            const int m = __reduce_max_sync(0xFFFFFFFFu, qn);
                            for (int i = 0; i < m; ++i) {
                                const bool on = i < qn;
                                list_insert<RKN>(top, topp, on ? hk[i * kRows] : 0ull, on ? hp[i * kRows] : 0.f, on);
                            }
                        }
                        qn = 0;
                    }
                    const float s = __uint_as_float(sv[j]);
                    float gs = s;
#pragma unroll
                    for (int o = 1; o < G; o <<= 1) gs += __shfl_xor_sync(0xFFFFFFFFu, gs, o);
                    const int c = c0 + 32 * half + j;
                    const bool cand = valid && c < ci && p.k > 0;
                    if (RK > 0) {
                        const uint64_t key = make_key(gs * sc_g, c);
                        if (cand && key > top[RKN - 1]) {
                            hk[qn * kRows] = key;
                            hp[qn * kRows] = s * p.scale;
                            ++qn;
                        }
                    } else if (cand) {
                        const uint64_t key = make_key(gs * sc_g, c);
                        if (key > hk[0]) sift_down_p(hk, hp, p.k, key, s * p.scale);
                    }
                    if (c == ci) own = s * p.scale;
                }
                if (RK > 0) {
                    // insert the queued keys: as many network passes as the warp's longest queue (the loop
                    // above inserted and emptied the queue after its first kQueue candidates)
                    const int m = __reduce_max_sync(0xFFFFFFFFu, qn);
                    for (int i = 0; i < m; ++i) {
                        const bool on = i < qn;
                        list_insert<RKN>(top, topp, on ? hk[i * kRows] : 0ull, on ? hp[i * kRows] : 0.f, on);
                    }
                }
            }
        }
        if (ok && valid) {
            const size_t row_g = (((size_t)b * p.Hkv + g) * p.N) + q0 + qi;
            const size_t row_h = (((size_t)b * p.H + (size_t)g * G + h) * p.N) + q0 + qi;
            const int ns = p.k + 1;
            if (RK > 0) {
                // the list is already in descending key order
#pragma unroll
                for (int j = 0; j < RKN; ++j) {
                    if (j < p.k) {
                        if (h == 0) sel_idx[row_g * p.k + j] = key_index(top[j]);
                        sel_score[row_h * ns + j] = top[j] ? topp[j] : -INFINITY;
                    }
                }
            } else {
                // heap sort: slots 0..k-1 end in descending key order
                for (int n = p.k; n > 1; --n) {
                    const uint64_t top0 = hk[0];
                    const float topp0 = hp[0];
                    sift_down_p(hk, hp, n - 1, hk[(n - 1) * kRows], hp[(n - 1) * kRows]);
                    hk[(n - 1) * kRows] = top0;
                    hp[(n - 1) * kRows] = topp0;
                }
                if (h == 0)
                    for (int j = 0; j < p.k; ++j) sel_idx[row_g * p.k + j] = key_index(hk[j * kRows]);
                for (int j = 0; j < p.k; ++j) sel_score[row_h * ns + j] = hk[j * kRows] ? hp[j * kRows] : -INFINITY;
            }
            sel_score[row_h * ns + p.k] = own;
        }
        (void)own_s;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

int stages_for(int k) { return k <= 32 ? 2 : 4; }

// Test control: HILS_SELECT_RESIDENT=0 keeps the per-row lists of the streaming epilogue.
bool res_disabled()
{
    const char *v = getenv("HILS_SELECT_RESIDENT");
    return v && strcmp(v, "0") == 0;
}

int max_tiles(const Dims &p) { return (int)(((long long)p.q_offset + p.N - 1) / p.C / kTile) + 1; }

}  // namespace

// Every tile of a CTA resident in TMEM (at most 8 tiles of 64 columns), register lists (k <= 16), and
// two or more heads per group to split the columns.
bool select_tc_resident(const Dims &p) { return p.k <= 16 && p.G >= 2 && max_tiles(p) <= 8 && !res_disabled(); }

namespace {

template <int G>
cudaError_t launch_g(const Dims &p, const void *Q, const void *L, int32_t *sel_idx, float *sel_score,
                     const DeviceCtl &ctl, cudaStream_t s)
{
    constexpr int BQ = kRows / G;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    CUtensorMap tl;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)p.B * p.Hkv * p.nL};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    const cuuint32_t es[2] = {1, 1};
    if (fn(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(L), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int nsl = stages_for(p.k);
    const int rk = p.k <= 16 ? 16 : 0;   // register list for k <= 16, shared-memory heap above
    size_t smem = make_layout(rk ? kQueue : p.k, nsl).total + 1024;
    dim3 grid((p.N + BQ - 1) / BQ, p.Hkv, p.B);
    const int n_tiles_max = max_tiles(p);
    const bool res = select_tc_resident(p);
    uint32_t tcols = kTmemCols;
    if (res) {
        while (tcols < (uint32_t)n_tiles_max * kTile) tcols <<= 1;
        if (tcols > 256 && smem < 120 * 1024) smem = 120 * 1024;   // 512 columns: one CTA per SM
    }
    cudaError_t e;
#define HILS_LAUNCH_SEL(NS, RKV, RESV)                                                                       \
    {                                                                                                        \
        auto kern = select_tc_kernel<G, NS, RKV, RESV>;                                                      \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);              \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, kThreads, smem, s>>>(tl, p, static_cast<const __nv_bfloat16 *>(Q), sel_idx, sel_score,  \
                                          ctl.status, (unsigned long long)ctl.wait_limit, tcols);            \
    }
    if (rk && res) HILS_LAUNCH_SEL(2, 16, G >= 2)
    else if (rk) HILS_LAUNCH_SEL(2, 16, false)
    else if (nsl == 2) HILS_LAUNCH_SEL(2, 0, false)
    else HILS_LAUNCH_SEL(4, 0, false)
#undef HILS_LAUNCH_SEL
    return cudaGetLastError();
}

}  // namespace

bool select_tc_supported(const Dims &p, hils_dtype in)
{
    if (in != HILS_BF16 || p.d != kD || p.N < 2) return false;
    if (p.G != 1 && p.G != 2 && p.G != 4 && p.G != 8 && p.G != 16) return false;
    return make_layout(p.k, stages_for(p.k)).total + 1024 <= 227 * 1024;
}

cudaError_t launch_select_prefill_tc(const Dims &p, const void *Q, const void *L, int32_t *sel_idx,
                                     float *sel_score, const DeviceCtl &ctl, cudaStream_t s)
{
    switch (p.G) {
    case 1: return launch_g<1>(p, Q, L, sel_idx, sel_score, ctl, s);
    case 2: return launch_g<2>(p, Q, L, sel_idx, sel_score, ctl, s);
    case 4: return launch_g<4>(p, Q, L, sel_idx, sel_score, ctl, s);
    case 8: return launch_g<8>(p, Q, L, sel_idx, sel_score, ctl, s);
    default: return launch_g<16>(p, Q, L, sel_idx, sel_score, ctl, s);
    }
}

}  // namespace hils
