// select_prefill_q.cu -- landmark scoring and top-k chunk selection on the sm_100a tensor cores, one
// product row per query (bf16 in, d = 128, k <= 32).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Sec. 3 Methodology, "Sparse
// training": every query scores all chunk summaries and keeps the top-K; Sec. 4, "Architecture":
// under GQA the group's heads share one selection.
//
// The selection ranks chunks by the group score mean_h(scale q_h . L_c) = scale qbar . L_c with
// qbar = mean_h q_h, so one product row per query suffices (G times fewer rows than one per head).
// qbar is formed in float32 from the bf16 query rows and split into two bf16 parts, hi = bf16(qbar)
// and lo = bf16(qbar - hi), which hold it to 2^-17 relative; the product runs over K = 2d = 256 as
// [hi | lo] . [L_c | L_c], so the group score keeps float32 accuracy (about 1e-6) while both
// operands stay bf16.
//
// One CTA owns 128 consecutive queries of one kv-group.  Warp 0 streams the landmarks of chunks
// 0 .. c_hi through shared memory in tiles of 128 (TMA, 128-byte swizzle, no multicast) and issues
// one tcgen05.mma chain per tile (M = 128 queries, N = 128 chunks, K = 256) into one of two TMEM
// score buffers.  Warps 2..5, one thread per query, read the scores, and keep the row's k best
// (group score, chunk) keys as a sorted list in registers: a candidate that beats the list's last
// key is queued in shared memory, and the warp inserts the queued keys together with a branch-free
// network.  Ties go to the lower chunk index through the key order.  After the scan, the per-head
// scores of the k selected slots and the own chunk (the fusion scores the attention needs) are
// computed on CUDA cores from the query rows staged in shared memory.
//
// The same kernel serves the local window and the per-chunk bias of the retrieval score (Sec. 2
// Preliminary and Sec. 5 "Experimental setup": a chunk-aligned window of the own chunk and the wc - 1
// chunks before it is always attended, and retrieval ranks only the chunks before it; Sec. 3 "Linear
// surrogate for chunk mass": the bias of chunk c is added to every head's score of c): the candidates
// are c <= c_i - wc, the bias is added to each candidate's group score and to every slot score, and a
// row holds k + wc - 1 past slots (the retrieved chunks, then the window's past chunks ascending).
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kThreads = 320;          // warp 0 loads and issues, warp 1 holds TMEM, warps 2-9 rank
constexpr int kRows = 128;               // queries per CTA (MMA M)
constexpr int kD = 128;
constexpr int kTile = 128;               // landmarks per tile (MMA N)
constexpr uint32_t kTileBytes = kTile * kD * 2;
constexpr uint32_t kQbarBytes = 4 * 16384;   // [hi d0-63 | hi d64-127 | lo d0-63 | lo d64-127], 128 rows each
constexpr uint32_t kTmemCols = 256;      // two 128-column score buffers
constexpr int kQueue = 16;               // candidates queued per row between insertions
constexpr int kNSL = 2;                  // landmark tile stages
constexpr int kHeadBatch = 4;            // query heads staged at once for the slot scores
constexpr unsigned long long kDrainNs = 2000000000ull;
constexpr uint32_t IDESC = idesc_bf16_f32(128, kTile, false, false);

struct Layout {
    uint32_t qbar, l, bar, misc, queue, selc, total;
};

// Shared memory: qbar (64 KB), the landmark stages, barriers, the candidate queue, then the rows'
// selected chunks.  After the scan the first kQbarBytes + kNSL * kTileBytes bytes hold query rows.
__host__ __device__ inline Layout make_layout(int k, int wc = 1)
{
    Layout L;
    L.qbar = 0;
    L.l = kQbarBytes;
    L.bar = L.l + kNSL * kTileBytes;
    L.misc = L.bar + 16 * 8;
    L.queue = L.misc + 16;
    L.selc = L.queue + 2u * 8u * kQueue * kRows;   // one queue per (row, column half)
    L.total = L.selc + 4u * (uint32_t)(k + wc) * kRows;
    return L;
}
static_assert(kHeadBatch * kRows * kD * 2 <= kQbarBytes + kNSL * kTileBytes, "query rows fit the freed stages");

// Insert key x into the descending list a[0..RK) if it beats the last entry: every slot takes its
// own, its upper neighbour's or the new key from two comparisons, all at once.
template <int RK>
__device__ __forceinline__ void list_insert(uint64_t (&a)[RK], uint64_t x, bool on)
{
    bool gt[RK];
#pragma unroll
    for (int i = 0; i < RK; ++i) gt[i] = on && x > a[i];
#pragma unroll
    for (int i = RK - 1; i > 0; --i) a[i] = gt[i] ? (gt[i - 1] ? a[i - 1] : x) : a[i];
    a[0] = gt[0] ? x : a[0];
}

// Sort a[0..RK) (RK a power of two) into descending order: a bitonic network whose indices are all
// known at compile time, so the list stays in registers.
template <int RK>
__device__ __forceinline__ void list_sort_desc(uint64_t (&a)[RK])
{
#pragma unroll
    for (int size = 2; size <= RK; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
            for (int i = 0; i < RK; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    // blocks with (i & size) == 0 go descending, the others ascending; the last merge
                    // (size == RK) leaves everything descending
                    const bool desc = (i & size) == 0;
                    const bool swap = desc ? (a[i] < a[j]) : (a[i] > a[j]);
                    const uint64_t ki = a[i], kj = a[j];
                    a[i] = swap ? kj : ki;
                    a[j] = swap ? ki : kj;
                }
            }
        }
    }
}

template <int RK, bool BIAS>
__global__ void __launch_bounds__(kThreads, 1)
    select_q_kernel(const __grid_constant__ CUtensorMap tmL, Dims p, const __nv_bfloat16 *__restrict__ Q,
                    const __nv_bfloat16 *__restrict__ Lm, int32_t *__restrict__ sel_idx,
                    float *__restrict__ sel_score, int wc, const float *__restrict__ bias, unsigned int *status,
                    unsigned long long limit_ns)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Layout Ly = make_layout(p.k, wc);
    const int G = p.G, ns = p.k + wc, kp = p.k + wc - 1;   // slots per row; past slots per row

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q0 = blockIdx.x * kRows, g = blockIdx.y, b = blockIdx.z;
    const int nq = min(kRows, p.N - q0);
    const int c_hi = (int)(((long long)p.q_offset + q0 + nq - 1) / p.C);   // own chunk of the last query
    // candidates are chunks c <= c_i - wc <= c_hi - wc; without any (k = 0, or the block's queries all
    // inside their first wc chunks) the scan is skipped and only the window's slot scores are written
    const int n_tiles = (p.k > 0 && c_hi - wc >= 0) ? (c_hi - wc) / kTile + 1 : 0;
    const int ksteps = G == 1 ? 8 : 16;   // with one head qbar = q is exact in bf16: lo = 0

    const uint32_t sQ = smem_addr(base + Ly.qbar), sL = smem_addr(base + Ly.l), bar0 = smem_addr(base + Ly.bar);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + Ly.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 8);
    uint64_t *queue = reinterpret_cast<uint64_t *>(base + Ly.queue);
    int *selc = reinterpret_cast<int *>(base + Ly.selc);
    const float *bias_bg = BIAS ? bias + ((size_t)b * p.Hkv + g) * p.nL : nullptr;
    auto L_FULL = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto L_EMPTY = [&](int s) { return bar0 + 8u * (uint32_t)(kNSL + s); };
    auto S_FULL = [&](int s) { return bar0 + 8u * (uint32_t)(2 * kNSL + s); };
    auto S_FREE = [&](int s) { return bar0 + 8u * (uint32_t)(2 * kNSL + 2 + s); };
    const uint32_t MMA_DONE = bar0 + 8u * (uint32_t)(2 * kNSL + 4);

    if (tid == 0) {
        for (int s = 0; s < kNSL; ++s) {
            mbar_init(L_FULL(s), 1);
            mbar_init(L_EMPTY(s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(S_FULL(s), 1);
            mbar_init(S_FREE(s), 8);
        }
        mbar_init(MMA_DONE, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tensormap(&tmL);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), kTmemCols);
        tmem_relinquish();
    }
    // qbar of each query row.  The G heads' rows are copied to shared memory (asynchronous 16-byte
    // copies, kHeadBatch heads at a time, into the space the landmark stages use later), summed in
    // float32 per (row, 16-byte piece), and the mean is split into bf16 hi and lo and written in the
    // 128-byte-swizzled K-major layout the MMA reads (row r = query, piece j of a 64-column half at
    // j ^ (r % 8))
    {
        constexpr int NIT = (kRows * 16 + kThreads - 1) / kThreads;
        float acc[NIT][8];
#pragma unroll
        for (int u = 0; u < NIT; ++u)
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[u][x] = 0.f;
        unsigned char *stage = base;   // [head in batch][query][16 pieces]
        for (int h0 = 0; h0 < G; h0 += kHeadBatch) {
            const int hb = min(kHeadBatch, G - h0);
            for (int e = tid; e < hb * nq * 16; e += kThreads) {
                const int hh = e / (nq * 16), rem = e % (nq * 16), qi = rem >> 4, seg = rem & 15;
                const __nv_bfloat16 *src =
                    Q + ((((size_t)b * p.H + (size_t)g * G + h0 + hh) * p.N) + q0 + qi) * kD + seg * 8;
                const uint32_t dst = smem_addr(stage + (((size_t)hh * kRows + qi) * 16 + seg) * 16);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
            }
            asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
            __syncthreads();
#pragma unroll
            for (int u = 0; u < NIT; ++u) {
                const int e = tid + u * kThreads, r = e >> 4, seg = e & 15;
                if (e < kRows * 16 && r < nq) {
                    for (int hh = 0; hh < hb; ++hh) {
                        float f[8];
                        unpack_bf16x8(*reinterpret_cast<const uint4 *>(stage + (((size_t)hh * kRows + r) * 16 + seg) * 16),
                                      f);
#pragma unroll
                        for (int x = 0; x < 8; ++x) acc[u][x] += f[x];
                    }
                }
            }
            __syncthreads();
        }
        const float inv_g = 1.0f / (float)G;
#pragma unroll
        for (int u = 0; u < NIT; ++u) {
            const int e = tid + u * kThreads, r = e >> 4, seg = e & 15;
            if (e >= kRows * 16) continue;
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float m0 = acc[u][2 * x] * inv_g, m1 = acc[u][2 * x + 1] * inv_g;
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(m0, m1);
                const __nv_bfloat162 l2 = __floats2bfloat162_rn(m0 - __low2float(h2), m1 - __high2float(h2));
                hi[x] = *reinterpret_cast<const uint32_t *>(&h2);
                lo[x] = *reinterpret_cast<const uint32_t *>(&l2);
            }
            const uint32_t off =
                (uint32_t)(seg >> 3) * 16384u + (uint32_t)r * 128u + (uint32_t)(((seg & 7) ^ (r & 7)) << 4);
            *reinterpret_cast<uint4 *>(base + Ly.qbar + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(base + Ly.qbar + 2 * 16384u + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
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
                while (next < n_tiles && next <= t + kNSL - 1) {
                    const int st = next % kNSL;
                    if (next >= kNSL &&
                        !mbar_wait(L_EMPTY(st), (uint32_t)(((next / kNSL) - 1) & 1), limit_ns, abort_flag, status)) {
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
                const int st = t % kNSL;
                if (!mbar_wait(L_FULL(st), (uint32_t)((t / kNSL) & 1), limit_ns, abort_flag, status)) break;
                if (t >= 2 && !mbar_wait(S_FREE(t & 1), (uint32_t)(((t >> 1) - 1) & 1), limit_ns, abort_flag, status))
                    break;
                tc_fence_after();
                const uint32_t la = sL + (uint32_t)st * kTileBytes;
                for (int s = 0; s < ksteps; ++s)
                    mma_bf16_ss(tmem + (uint32_t)(t & 1) * kTile,
                                smem_desc_sw128(sQ + (uint32_t)(s >> 2) * 16384u + (uint32_t)(s & 3) * 32u, 16, 1024),
                                smem_desc_sw128(la + (uint32_t)((s >> 2) & 1) * (kTileBytes / 2) + (uint32_t)(s & 3) * 32u,
                                                16, 1024),
                                IDESC, s > 0 ? 1u : 0u);
                mma_commit(S_FULL(t & 1));
                mma_commit(L_EMPTY(st));
            }
            mma_commit(MMA_DONE);
            mbar_drain(MMA_DONE, 0, kDrainNs);
            for (int u = max(0, next - kNSL); u < next; ++u)
                mbar_drain(L_FULL(u % kNSL), (uint32_t)((u / kNSL) & 1), kDrainNs);
        }
        __syncwarp();
    } else if (warp >= 2) {
        // two warps per quarter of the rows (TMEM lanes 32 qq ..): warps 2-5 rank the first two 32-column
        // parts of every tile, warps 6-9 the last two; their lists merge after the scan
        const int qq = warp & 3, ch = (warp - 2) >> 2;
        const int r = 32 * qq + lane;
        const bool valid = r < nq;
        const long long pos = (long long)p.q_offset + q0 + r;
        const int ci = (int)(pos / p.C);
        const int c_lim = ci - wc + 1;   // candidates c < c_lim
        const uint32_t trow = tmem + ((uint32_t)(32 * qq) << 16);
        uint64_t *hk = queue + (size_t)ch * kQueue * kRows + r;
        uint64_t top[RK];
#pragma unroll
        for (int i = 0; i < RK; ++i) top[i] = 0ull;
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            int w_ok = 1;
            if (lane == 0) w_ok = mbar_wait(S_FULL(t & 1), (uint32_t)((t >> 1) & 1), limit_ns, abort_flag, status);
            if (!__shfl_sync(0xFFFFFFFFu, w_ok, 0)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int part = 2 * ch; part < 2 * ch + 2; ++part) {
                uint32_t sv[32];
                tmem_ld32(trow + (uint32_t)(t & 1) * kTile + 32u * part, sv);
                tmem_wait_ld();
                if (part == 2 * ch + 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(S_FREE(t & 1));
                }
                const int cb = t * kTile + 32 * part;
                float bv[BIAS ? 32 : 1];   // the 32 chunks' biases (the same address in every lane: broadcast)
                if constexpr (BIAS) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) bv[j] = cb + j < p.nL ? __ldg(bias_bg + cb + j) : 0.f;
                }
                int qn = 0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (j == kQueue) {
                        // the queue is full after kQueue candidates: insert them before going on.  The
                        // very first time the list is still empty: the queued keys are copied in and
                        // sorted by a network instead of inserted one by one.
                        if (t == 0 && part == 2 * ch) {
#pragma unroll
                            for (int i = 0; i < RK; ++i) top[i] = (i < kQueue && i < qn) ? hk[i * kRows] : 0ull;
                            list_sort_desc<RK>(top);
                        } else {
                            const int m = __reduce_max_sync(0xFFFFFFFFu, qn);
                            for (int i = 0; i < m; ++i) {
                                const bool on = i < qn;
                                list_insert<RK>(top, on ? hk[i * kRows] : 0ull, on);
                            }
                        }
                        qn = 0;
                    }
                    const int c = cb + j;
                    float sc = __uint_as_float(sv[j]) * p.scale;
                    if constexpr (BIAS) sc += bv[j];
                    const uint64_t key = make_key(sc, c);
                    if (valid && c < c_lim && key > top[RK - 1]) {
                        hk[qn * kRows] = key;
                        ++qn;
                    }
                }
                const int m = __reduce_max_sync(0xFFFFFFFFu, qn);
                for (int i = 0; i < m; ++i) {
                    const bool on = i < qn;
                    list_insert<RK>(top, on ? hk[i * kRows] : 0ull, on);
                }
            }
        }
        if (!ok) *abort_flag = 1;
        // the two column halves' lists of each row into one, kept by the first warp of the pair: the
        // second one's list goes through the queue space, free once every epilogue warp has finished
        // its scan (named barrier 2: the eight epilogue warps)
        uint64_t *xl = queue + r;   // [RK][kRows]
        asm volatile("bar.sync 2, 256;" ::: "memory");
        if (ch == 1) {
#pragma unroll
            for (int i = 0; i < RK; ++i) xl[i * kRows] = top[i];
        }
        asm volatile("bar.sync 2, 256;" ::: "memory");
        if (ch == 0) {
            // both lists descending: the elementwise maximum against the other list reversed is bitonic
            // and holds the RK largest; a merge network sorts it
#pragma unroll
            for (int i = 0; i < RK; ++i) {
                const uint64_t x = xl[(RK - 1 - i) * kRows];
                top[i] = top[i] > x ? top[i] : x;
            }
#pragma unroll
            for (int stride = RK / 2; stride > 0; stride >>= 1)
#pragma unroll
                for (int i = 0; i < RK; ++i)
                    if ((i & stride) == 0) {
                        const uint64_t a = top[i], c2 = top[i + stride];
                        top[i] = a > c2 ? a : c2;
                        top[i + stride] = a > c2 ? c2 : a;
                    }
        }
        // the selection: chunk indices in rank order (k < RK: the list's first k keys), then the window's
        // past chunks ascending, own chunk last
        if (valid && ch == 0) {
            const size_t row_g = (((size_t)b * p.Hkv + g) * p.N) + q0 + r;
#pragma unroll
            for (int j = 0; j < RK; ++j) {
                if (j < p.k) {
                    const int c = key_index(top[j]);
                    sel_idx[row_g * kp + j] = c;
                    selc[r * ns + j] = c;
                }
            }
            for (int j = p.k; j < kp; ++j) {
                const int c = ci - wc + 1 + (j - p.k);
                sel_idx[row_g * kp + j] = c >= 0 ? c : -1;
                selc[r * ns + j] = c >= 0 ? c : -1;
            }
            selc[r * ns + kp] = ci;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (*abort_flag) return;

    // ---- per-head slot scores: scale q_h . L_c for the k selected chunks and the own chunk ------------
    // query rows of up to kHeadBatch heads at a time in the freed stages (bf16, asynchronous copies),
    // 16-byte pieces rotated by query so that threads of different queries read different banks; one
    // thread per (query, slot), the next item's landmark row loaded while the current one is computed
    unsigned char *qrows = base;   // [head in batch][query][16 pieces] (uint4)
    const __nv_bfloat16 *Lbg = Lm + ((size_t)b * p.Hkv + g) * p.nL * kD;
    const int n_items = nq * ns;
    for (int h0 = 0; h0 < G; h0 += kHeadBatch) {
        const int hb = min(kHeadBatch, G - h0);
        if (h0 > 0) __syncthreads();
        for (int e = tid; e < hb * nq * 16; e += kThreads) {
            const int hh = e / (nq * 16), rem = e % (nq * 16), qi = rem >> 4, seg = rem & 15;
            const __nv_bfloat16 *src =
                Q + ((((size_t)b * p.H + (size_t)g * G + h0 + hh) * p.N) + q0 + qi) * kD + seg * 8;
            const uint32_t dst = smem_addr(qrows + (((size_t)hh * kRows + qi) * 16 + ((seg + qi) & 15)) * 16);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
        }
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        __syncthreads();
        uint4 nxt[16];
        auto fetch = [&](int it) {
            const int c = it < n_items ? selc[(it / ns) * ns + it % ns] : -1;
            const uint4 *lr = reinterpret_cast<const uint4 *>(Lbg + (size_t)(c >= 0 ? c : 0) * kD);
#pragma unroll
            for (int seg = 0; seg < 16; ++seg) nxt[seg] = (c >= 0) ? __ldg(lr + seg) : make_uint4(0u, 0u, 0u, 0u);
        };
        fetch(tid);
        for (int it = tid; it < n_items; it += kThreads) {
            uint4 lv[16];
#pragma unroll
            for (int seg = 0; seg < 16; ++seg) lv[seg] = nxt[seg];
            fetch(it + kThreads);
            const int qi = it / ns, j = it % ns;
            const int c = selc[qi * ns + j];
            float acc[kHeadBatch];
#pragma unroll
            for (int hh = 0; hh < kHeadBatch; ++hh) acc[hh] = 0.f;
#pragma unroll
            for (int seg = 0; seg < 16; ++seg) {
                float lf[8];
                unpack_bf16x8(lv[seg], lf);
#pragma unroll
                for (int hh = 0; hh < kHeadBatch; ++hh) {
                    if (hh < hb) {
                        float qf[8];
                        unpack_bf16x8(*reinterpret_cast<const uint4 *>(
                                          qrows + (((size_t)hh * kRows + qi) * 16 + ((seg + qi) & 15)) * 16),
                                      qf);
#pragma unroll
                        for (int x = 0; x < 8; ++x) acc[hh] = fmaf(qf[x], lf[x], acc[hh]);
                    }
                }
            }
#pragma unroll
            for (int hh = 0; hh < kHeadBatch; ++hh) {
                if (hh < hb) {
                    const size_t row_h = (((size_t)b * p.H + (size_t)g * G + h0 + hh) * p.N) + q0 + qi;
                    sel_score[row_h * ns + j] =
                        c >= 0 ? acc[hh] * p.scale + (BIAS ? __ldg(bias_bg + c) : 0.f) : -INFINITY;
                }
            }
        }
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

}  // namespace

// The kernel with one row per query pays for its G-fold smaller scan with the per-head slot scores it
// computes afterwards on CUDA cores; the kernel with one row per head gets those with the scan.  So
// this one is used where the scan dominates: k above 16 (the other kernel keeps larger lists in a
// shared-memory heap) or more than 512 visible chunks.
bool select_q_supported(const Dims &p, hils_dtype in, int wc)
{
    if (in != HILS_BF16 || p.d != kD || p.N < 2 || p.k > 32 || wc < 1) return false;
    return make_layout(p.k, wc).total + 1024 <= 227 * 1024;
}

bool select_q_preferred(const Dims &p)
{
    const long long c_max = ((long long)p.q_offset + p.N - 1) / p.C;
    return p.k > 16 || c_max >= 512;
}

cudaError_t launch_select_prefill_q(const Dims &p, const void *Q, const void *L, int32_t *sel_idx, float *sel_score,
                                    const DeviceCtl &ctl, cudaStream_t s, int wc, const float *bias)
{
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
    const size_t smem = make_layout(p.k, wc).total + 1024;
    dim3 grid((p.N + kRows - 1) / kRows, p.Hkv, p.B);
    cudaError_t e;
#define HILS_LAUNCH_SELQ(RKV, BV)                                                                            \
    {                                                                                                        \
        auto kern = select_q_kernel<RKV, BV>;                                                                \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);              \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, kThreads, smem, s>>>(tl, p, static_cast<const __nv_bfloat16 *>(Q),                      \
                                          static_cast<const __nv_bfloat16 *>(L), sel_idx, sel_score, wc,     \
                                          bias, ctl.status, (unsigned long long)ctl.wait_limit);             \
    }
    if (p.k <= 16) {
        if (bias) HILS_LAUNCH_SELQ(16, true) else HILS_LAUNCH_SELQ(16, false)
    } else {
        if (bias) HILS_LAUNCH_SELQ(32, true) else HILS_LAUNCH_SELQ(32, false)
    }
#undef HILS_LAUNCH_SELQ
    return cudaGetLastError();
}

}  // namespace hils
