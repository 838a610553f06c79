// attend_prefill_tc_persistent.cu -- the tensor-core chunk attention as a persistent kernel: one CTA per SM
// walks query tiles back to back, building the next tile's chunk union while the current tile's last
// products run (bf16 in, d = 128, C = 64).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1):
//   Abstract / Sec. 3 "Hierarchical softmax": softmax inside every selected
//   chunk, chunk outputs fused by a softmax over the retrieval scores;
//   Sec. 4 "Kernel design": adjacent queries share most of their chunks, so a
//   block of M queries is processed over the union of their chunks, making the
//   tensor-core product (M x G, d) x (d, S) and loading each chunk once;
//   Sec. 4 "Architecture": a GQA group's heads share the retrieved chunks.
//
// One CTA owns 128 rows = (128 / G) consecutive queries x the G heads of one
// kv-group (row r = query * G + head, so that a warp's 32 rows cover 32 / G
// whole queries and can skip a chunk none of them selected).  It walks the union of the
// chunks its queries selected, in ascending chunk order, with warp-specialised
// roles that meet on mbarriers:
//   warp 0 (one thread)  TMA loads of Q once and of the union's K tiles, two
//                        chunks per ring slot (128-byte swizzle, no multicast);
//   warp 1 (one thread)  TMA loads of the V tiles, two chunks per ring slot;
//                        the warp also owns the TMEM allocation;
//   warp 2 (one thread)  tcgen05.mma issue of S = Q K^T (bf16, A and B from
//                        shared memory) on two chunks at once (N = 128, the
//                        tensor core's efficient width) into one of two TMEM
//                        S buffers;
//   warp 3 (one thread)  tcgen05.mma issue of O += P V (f16 or bf16, P from
//                        TMEM, V from shared memory) on the same pairs (K = 128 keys);
//                        two issuers keep the tensor core busy while either
//                        one waits;
//   warps 4..15          three groups of four warps, one thread per row; group
//                        t % 3 handles chunk t: it reads S from TMEM (and frees
//                        the S buffer at once), takes the softmax over the
//                        chunk's visible keys, scales it by the row's fusion
//                        weight (0 if the row's query did not select the chunk)
//                        and writes P (16-bit) to its half of a TMEM P buffer.  At
//                        the end the groups read O from TMEM and store it.
// Because each chunk's softmax is normalised on its own and the fusion weights
// are known before the loop, P already carries w_c / l_c and the accumulator
// needs no rescaling between chunks.
//
// Value product precision, as in the per-tile kernel: a streaming pass converts
// V to f16 once per call and flags every (b, kv-head) slice holding a value of
// magnitude >= 65536; a tile of an unflagged slice reads the f16 copy and rounds
// P to f16 (relative 2^-11), a tile of a flagged slice reads V as given and
// rounds P to bf16, so V always enters the product exactly.
//
// Every barrier wait is bounded: on expiry the CTA records HILS_ERR_TIMEOUT,
// stops issuing work, waits (with its own bound) for the copies and MMAs it has
// in flight, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_fp16.h>

#include "chunk_softmax.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kGroups = 3;        // softmax warp groups (4 warps each); group t % kGroups handles chunk t
constexpr int kThreads = 128 + 128 * kGroups;   // K loads, V loads + TMEM, QK issue, PV issue, softmax groups
constexpr int kSM = 128 * kGroups;              // softmax threads
constexpr int kRows = 128;        // MMA M
constexpr int kChunk = 64;        // C
constexpr int kD = 128;           // d
constexpr int kSP = 2;                // S buffers (a pair of chunks, 128 columns each) = key ring slots
constexpr int kPB = 2;                // P buffers (a pair of chunks, 64 columns each)
constexpr uint32_t kTmemCols = 512;   // S pair buffers (2 x 128 columns), O (128), up to 2 P pair buffers (64 each)
constexpr uint32_t kColO = 256, kColP = 384;
constexpr uint32_t kPairBytes = 32768;   // K and V ring slots: [c0 d0-63 | c1 d0-63 | c0 d64-127 | c1 d64-127]
constexpr unsigned long long kDrainNs = 2000000000ull;
constexpr int kPolyPairEvery = 4; // exponential pairs computed by exp2_poly_x2: 1 in kPolyPairEvery

constexpr uint32_t IDESC_QK2 = idesc_bf16_f32(128, 128, false, false);  // S = Q K^T over two chunks, K-major
constexpr uint32_t IDESC_QK1 = idesc_bf16_f32(128, 64, false, false);   // the same for a lone last chunk
constexpr uint32_t IDESC_PV = idesc_f16_f32(128, 128, false, true);    // O += P V, f16, V MN-major
constexpr uint32_t IDESC_PV_BF16 = idesc_bf16_f32(128, 128, false, true);   // the same in bf16 (wide slices)

struct Layout {
    uint32_t q, k, v, bar, misc, bitmap, uni0, uni1, selbuf, scbuf, qlist, qslot, qcnt, wts, total;
};

__host__ __device__ inline uint32_t al16(uint32_t x) { return (x + 15u) & ~15u; }

constexpr int kMaxBars = 64;

// Shared memory: Q (32 KB), kSP key slots and NSV value slots (two chunks, 32 KB each), barriers, then
// the selection bookkeeping: the chunk union of two tiles (the current one and the next, built while
// the current one's last products run) and one copy of the rest (rebuilt between tiles).
__host__ __device__ inline Layout make_layout(int nsk, int nsv, int k, int nwords, int BQ)
{
    Layout L;
    const uint32_t ns = (uint32_t)(k + 1);
    L.q = 0;
    L.k = 32768;
    L.v = L.k + (uint32_t)nsk * kPairBytes;
    L.bar = L.v + (uint32_t)nsv * kPairBytes;
    L.misc = L.bar + kMaxBars * 8;
    L.bitmap = L.misc + 16;
    L.uni0 = al16(L.bitmap + 4u * (uint32_t)nwords);
    L.uni1 = al16(L.uni0 + 4u * ns * (uint32_t)BQ);
    L.selbuf = al16(L.uni1 + 4u * ns * (uint32_t)BQ);              // the tile's sel_idx rows
    L.scbuf = al16(L.selbuf + 4u * (uint32_t)k * (uint32_t)BQ);    // the rows' sel_score values
    L.qlist = al16(L.scbuf + 4u * ns * (uint32_t)kRows);
    L.qslot = al16(L.qlist + 4u * ns * (uint32_t)BQ);
    L.qcnt = al16(L.qslot + 4u * ns * (uint32_t)BQ);
    L.wts = al16(L.qcnt + 4u * (uint32_t)BQ);
    L.total = al16(L.wts + 4u * ns * (uint32_t)kRows);
    return L;
}

// Barrier slots.  Pairs are numbered across the CTA's tiles (g = pairs of earlier tiles + pair in
// tile).  Key slot / S buffer and P buffer: g % 2; value slot: g % NSV.
//   K_LAND[b], QK_READY[b], QK_DONE[b], V_LAND[v], PV_READY[b], PV_DONE[b] as in the one-tile kernel
//   Q_FULL      Q of tile i has landed (phase i)
//   O_FULL      every value product of tile i is complete (phase i)
//   O_EMPTY     the softmax warps have read O of tile i out of TMEM (12 arrivals; phase i)
//   BOOK[j]     the bookkeeping of tile i (j = i % 2) is built (phase i / 2)
template <int NSV>
struct Bars {
    static constexpr int Q_FULL = 0, K_LAND = 1, QK_READY = K_LAND + kSP, QK_DONE = QK_READY + kSP,
                         V_LAND = QK_DONE + kSP, PV_READY = V_LAND + NSV, PV_DONE = PV_READY + kPB,
                         O_FULL = PV_DONE + kPB, O_EMPTY = O_FULL + 1, BOOK = O_EMPTY + 1,
                         MMA_DONE = BOOK + 2;   // MMA_DONE + 0/1: the two issuers
    static_assert(MMA_DONE + 1 < kMaxBars, "barrier slots");
};

__device__ __forceinline__ void store_row32(float *dst, const uint32_t *v)
{
#pragma unroll
    for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(dst + i) =
            make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                        __uint_as_float(v[i + 3]));
}

__device__ __forceinline__ void store_row32(__nv_bfloat16 *dst, const uint32_t *v)
{
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        uint4 u;
        __nv_bfloat162 a = __floats2bfloat162_rn(__uint_as_float(v[i]), __uint_as_float(v[i + 1]));
        __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        __nv_bfloat162 c = __floats2bfloat162_rn(__uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
        __nv_bfloat162 d = __floats2bfloat162_rn(__uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
        u.x = *reinterpret_cast<uint32_t *>(&a);
        u.y = *reinterpret_cast<uint32_t *>(&b);
        u.z = *reinterpret_cast<uint32_t *>(&c);
        u.w = *reinterpret_cast<uint32_t *>(&d);
        *reinterpret_cast<uint4 *>(dst + i) = u;
    }
}

// lane 0 waits, the result is broadcast so the warp decides uniformly
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, unsigned long long lim, volatile int *abort_flag,
                                          unsigned int *status)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, lim, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

__device__ __forceinline__ void mbar_arrive_n(uint32_t bar, uint32_t n)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(n) : "memory");
}

// 4-byte global -> shared copy that completes asynchronously (waited for by cp_async_wait_all)
__device__ __forceinline__ void cp_async4(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Named barrier 1 over the softmax warps; bar_red_or returns whether any of them passed a true flag.
__device__ __forceinline__ void sm_sync() { asm volatile("bar.sync 1, %0;" ::"r"(32 * 4 * kGroups) : "memory"); }
__device__ __forceinline__ bool sm_sync_any(bool flag)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)flag), "r"(32 * 4 * kGroups)
                 : "memory");
    return r != 0;
}

// One loader thread streams the n pair tiles of one query tile through a ring of `slots` buffers.
// Pair j of the tile is pair base + j of the CTA: it goes to slot (base + j) % slots once the pair
// that last used the slot is complete (completion barriers `done` go by pair % 2), lands on `land`
// (by slot) and is then announced on `ready` (by pair % 2).  Up to `slots` pairs are in flight.
// On an abort the thread waits, with its own bound, for the copies it started.  Returns false then.
template <typename Issue>
__device__ __forceinline__ bool stream_ring(int n, int base, int slots, uint32_t done0, uint32_t land0, uint32_t ready0,
                                            Issue &&issue, unsigned long long limit_ns, volatile int *abort_flag,
                                            unsigned int *status)
{
    int issued = 0, landed = 0;
    long long t_prog = cycle_now();
    bool ok = true;
    while (landed < n) {
        const int gi = base + issued;
        const int freed = gi - slots;
        if (issued < n && issued < landed + slots &&
            (freed < 0 || mbar_test(done0 + 8u * (uint32_t)(freed & 1), (uint32_t)((freed >> 1) & 1)))) {
            issue(issued, gi % slots);
            ++issued;
            t_prog = cycle_now();
            continue;
        }
        const int gl = base + landed;
        const uint32_t lbar = land0 + 8u * (uint32_t)(gl % slots);
        const uint32_t lphase = (uint32_t)((gl / slots) & 1);
        if (landed < issued && mbar_test(lbar, lphase)) {
            mbar_arrive(ready0 + 8u * (uint32_t)(gl & 1));
            ++landed;
            t_prog = cycle_now();
            continue;
        }
        if (*abort_flag) {
            ok = false;
            break;
        }
        if (*reinterpret_cast<volatile unsigned int *>(status) != 0u) {
            *abort_flag = 1;
            ok = false;
            break;
        }
        if (past_limit(t_prog, limit_ns)) {
            *abort_flag = 1;
            atomicExch(status, 4u /* HILS_ERR_TIMEOUT */);
            ok = false;
            break;
        }
        if (landed < issued) mbar_try_wait_sleep(lbar, lphase, 200u);
        else mbar_try_wait_sleep(done0 + 8u * (uint32_t)(freed & 1), (uint32_t)((freed >> 1) & 1), 200u);
    }
    if (!ok)   // the copies must land before the CTA exits
        for (int v = landed; v < issued; ++v) {
            const int gv = base + v;
            mbar_drain(land0 + 8u * (uint32_t)(gv % slots), (uint32_t)((gv / slots) & 1), kDrainNs);
        }
    return ok;
}

// Query tile tau of the launch: the same order as a grid of (query tiles, kv-groups, batch) with the
// later (heavier) query tiles first.
struct TileId {
    int q0, g, b, nq;
};

__device__ __forceinline__ TileId tile_of(int tau, int tiles_x, const Dims &p, int BQ)
{
    TileId t;
    const int x = tau % tiles_x, rest = tau / tiles_x;
    t.g = rest % p.Hkv;
    t.b = rest / p.Hkv;
    t.q0 = (tiles_x - 1 - x) * BQ;
    t.nq = min(BQ, p.N - t.q0);
    return t;
}

template <int G, typename Tout, int NSV>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVb, Dims p,
                                const int32_t *__restrict__ sel_idx, const float *__restrict__ sel_score,
                                const unsigned int *__restrict__ wide_flags, Tout *__restrict__ O, unsigned int *status,
                                unsigned long long limit_ns, int nwords, int inject_stall, int n_tiles, int tiles_x)
{
    constexpr int BQ = kRows / G;
    using BR = Bars<NSV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Layout Ly = make_layout(kSP, NSV, p.k, nwords, BQ);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ns = p.k + 1;
    const int stride = (int)gridDim.x;

    const uint32_t sQ = smem_addr(base + Ly.q), sK = smem_addr(base + Ly.k), sV = smem_addr(base + Ly.v);
    const uint32_t bar0 = smem_addr(base + Ly.bar);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + Ly.misc);
    int *n_union_s = reinterpret_cast<int *>(base + Ly.misc + 4);        // [2]: misc + 4, misc + 8
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 12);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(base + Ly.bitmap);
    // the two chunk-union buffers, selected by tile parity (arithmetic, not an array of pointers)
    int *const uni0 = reinterpret_cast<int *>(base + Ly.uni0);
    const int uni_step = (int)((Ly.uni1 - Ly.uni0) / 4u);
    int *selbuf = reinterpret_cast<int *>(base + Ly.selbuf);
    float *scbuf = reinterpret_cast<float *>(base + Ly.scbuf);
    int *qlist = reinterpret_cast<int *>(base + Ly.qlist);
    int *qslot = reinterpret_cast<int *>(base + Ly.qslot);
    int *qcnt = reinterpret_cast<int *>(base + Ly.qcnt);
    float *wts = reinterpret_cast<float *>(base + Ly.wts);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };

    // ---- set-up: barriers and tensor memory, once per CTA ---------------------------------------
    if (tid == 0) {
        mbar_init(BAR(BR::Q_FULL), 1);
        for (int s = 0; s < kSP; ++s) {
            mbar_init(BAR(BR::K_LAND + s), 1);
            mbar_init(BAR(BR::QK_READY + s), 1 + 8);   // the key loader + 4 warps for each chunk of the pair
            mbar_init(BAR(BR::QK_DONE + s), 1);
            for (int a = 0; a < 8; ++a) mbar_arrive(BAR(BR::QK_READY + s));   // pairs 0, 1: S free
        }
        for (int s = 0; s < NSV; ++s) mbar_init(BAR(BR::V_LAND + s), 1);
        for (int s = 0; s < kPB; ++s) {
            mbar_init(BAR(BR::PV_READY + s), 1 + 8);   // the value loader + 4 warps for each chunk
            mbar_init(BAR(BR::PV_DONE + s), 1);
        }
        mbar_init(BAR(BR::O_FULL), 1);
        mbar_init(BAR(BR::O_EMPTY), 4 * kGroups);      // every softmax warp, after its epilogue reads
        mbar_init(BAR(BR::BOOK), 1);
        mbar_init(BAR(BR::BOOK + 1), 1);
        mbar_init(BAR(BR::MMA_DONE), 1);
        mbar_init(BAR(BR::MMA_DONE + 1), 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmVb);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ---------------- Q of each tile, then its key pairs ------------------------------------
        if (lane == 0) {
            int kp = 0, q_loads = 0;
            bool ok = true;
            for (int i = 0, tau = (int)blockIdx.x; ok && tau < n_tiles; ++i, tau += stride) {
                const TileId T = tile_of(tau, tiles_x, p, BQ);
                if (!mbar_wait(BAR(BR::BOOK + (i & 1)), (uint32_t)((i >> 1) & 1), limit_ns, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const int n_union = n_union_s[i & 1];
                const int *uni = uni0 + (i & 1) * uni_step;
                if (kp > 0 &&   // Q's buffer is free once the previous tile's last key product is complete
                    !mbar_wait(BAR(BR::QK_DONE + ((kp - 1) & 1)), (uint32_t)(((kp - 1) >> 1) & 1), limit_ns,
                               abort_flag, status)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(BAR(BR::Q_FULL), 32768u);
                tma_load_3d(sQ, &tmQ, BAR(BR::Q_FULL), 0, T.b * p.H + T.g * G, T.q0);
                tma_load_3d(sQ + 16384u, &tmQ, BAR(BR::Q_FULL), 64, T.b * p.H + T.g * G, T.q0);
                ++q_loads;
                const int kv_row0 = (T.b * p.Hkv + T.g) * p.T;
                const int n_pairs = (n_union + 1) >> 1;
                auto issue = [&](int pr, int st) {
                    const bool two = 2 * pr + 1 < n_union;
                    const uint32_t dst = sK + (uint32_t)st * kPairBytes;
                    mbar_arrive_expect_tx(BAR(BR::K_LAND + st), two ? 32768u : 16384u);
                    const int row0 = kv_row0 + uni[2 * pr] * kChunk;
                    tma_load_2d(dst, &tmK, BAR(BR::K_LAND + st), 0, row0);
                    tma_load_2d(dst + 16384u, &tmK, BAR(BR::K_LAND + st), 64, row0);
                    if (two) {
                        const int row1 = kv_row0 + uni[2 * pr + 1] * kChunk;
                        tma_load_2d(dst + 8192u, &tmK, BAR(BR::K_LAND + st), 0, row1);
                        tma_load_2d(dst + 24576u, &tmK, BAR(BR::K_LAND + st), 64, row1);
                    }
                };
                ok = stream_ring(n_pairs, kp, kSP, BAR(BR::QK_DONE), BAR(BR::K_LAND), BAR(BR::QK_READY), issue,
                                 limit_ns, abort_flag, status);
                kp += n_pairs;
            }
            if (q_loads > 0) mbar_drain(BAR(BR::Q_FULL), (uint32_t)((q_loads - 1) & 1), kDrainNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- value pairs ---------------------------------------------------------
        if (lane == 0) {
            int vp = 0;
            bool ok = true;
            for (int i = 0, tau = (int)blockIdx.x; ok && tau < n_tiles; ++i, tau += stride) {
                const TileId T = tile_of(tau, tiles_x, p, BQ);
                if (!mbar_wait(BAR(BR::BOOK + (i & 1)), (uint32_t)((i >> 1) & 1), limit_ns, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const int n_union = n_union_s[i & 1];
                const int *uni = uni0 + (i & 1) * uni_step;
                const int kv_row0 = (T.b * p.Hkv + T.g) * p.T;
                const int n_pairs = (n_union + 1) >> 1;
                // a slice whose values overflow f16 takes the bf16 value product (V as given)
                const CUtensorMap *tmVsel = __ldg(wide_flags + T.b * p.Hkv + T.g) != 0u ? &tmVb : &tmV;
                auto issue = [&](int pr, int st) {
                    const bool two = 2 * pr + 1 < n_union;
                    const uint32_t dst = sV + (uint32_t)st * kPairBytes;
                    mbar_arrive_expect_tx(BAR(BR::V_LAND + st), two ? 32768u : 16384u);
                    const int row0 = kv_row0 + uni[2 * pr] * kChunk;
                    tma_load_2d(dst, tmVsel, BAR(BR::V_LAND + st), 0, row0);
                    tma_load_2d(dst + 16384u, tmVsel, BAR(BR::V_LAND + st), 64, row0);
                    if (two) {
                        const int row1 = kv_row0 + uni[2 * pr + 1] * kChunk;
                        tma_load_2d(dst + 8192u, tmVsel, BAR(BR::V_LAND + st), 0, row1);
                        tma_load_2d(dst + 24576u, tmVsel, BAR(BR::V_LAND + st), 64, row1);
                    }
                };
                ok = stream_ring(n_pairs, vp, NSV, BAR(BR::PV_DONE), BAR(BR::V_LAND), BAR(BR::PV_READY), issue,
                                 limit_ns, abort_flag, status);
                vp += n_pairs;
            }
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3) {
        // ---------------- MMA issue: warp 2 the key products, warp 3 the value products ---------
        if (lane == 0) {
            const bool keys = (warp == 2);
            bool ok = true;
            if (keys && inject_stall) {
                // test control: wait once on a barrier nothing signals, so the bounded wait expires
                ok = mbar_wait(BAR(BR::MMA_DONE), 0, limit_ns, abort_flag, status);
            }
            uint64_t dq[8];
#pragma unroll
            for (int s = 0; s < 8; ++s) dq[s] = smem_desc_sw128(sQ + (s >> 2) * 16384u + (s & 3) * 32u, 16, 1024);
            int gp0 = 0;
            for (int i = 0, tau = (int)blockIdx.x; ok && tau < n_tiles; ++i, tau += stride) {
                const TileId T = tile_of(tau, tiles_x, p, BQ);
                const uint32_t idesc_pv = __ldg(wide_flags + T.b * p.Hkv + T.g) != 0u ? IDESC_PV_BF16 : IDESC_PV;
                if (!mbar_wait(BAR(BR::BOOK + (i & 1)), (uint32_t)((i >> 1) & 1), limit_ns, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const int n_union = n_union_s[i & 1];
                const int n_pairs = (n_union + 1) >> 1;
                if (keys && !mbar_wait(BAR(BR::Q_FULL), (uint32_t)(i & 1), limit_ns, abort_flag, status)) {
                    ok = false;
                    break;
                }
                for (int j = 0; ok && j < n_pairs; ++j) {
                    const int gp = gp0 + j;
                    if (!keys && j == 0 && i > 0 &&   // O of the previous tile has been read out
                        !mbar_wait(BAR(BR::O_EMPTY), (uint32_t)((i - 1) & 1), limit_ns, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = keys ? BAR(BR::QK_READY + (gp & 1)) : BAR(BR::PV_READY + (gp & 1));
                    const uint32_t phase = (uint32_t)((gp >> 1) & 1);
                    const long long t0 = cycle_now();
                    unsigned idle = 0;
                    while (!mbar_test(bar, phase)) {
                        if (*abort_flag) {
                            ok = false;
                            break;
                        }
                        if ((++idle & 63) == 0 && *reinterpret_cast<volatile unsigned int *>(status) != 0u) {
                            *abort_flag = 1;
                            ok = false;
                            break;
                        }
                        if (past_limit(t0, limit_ns)) {
                            *abort_flag = 1;
                            atomicExch(status, 4u /* HILS_ERR_TIMEOUT */);
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                    tc_fence_after();
                    if (keys) {
                        const uint32_t d_s = tmem + (uint32_t)(gp & 1) * 128u;
                        const uint64_t dk = smem_desc_sw128(sK + (uint32_t)(gp & 1) * kPairBytes, 16, 1024);
                        const uint32_t idesc = (2 * j + 1 < n_union) ? IDESC_QK2 : IDESC_QK1;
#pragma unroll
                        for (int s = 0; s < 8; ++s)
                            mma_bf16_ss(d_s, dq[s], dk + (uint64_t)(((s >> 2) * 16384u + (s & 3) * 32u) >> 4), idesc,
                                        s > 0 ? 1u : 0u);
                        mma_commit(BAR(BR::QK_DONE + (gp & 1)));
                    } else {
                        const uint32_t pa = tmem + kColP + (uint32_t)(gp & 1) * 64u;
                        const uint64_t dv = smem_desc_sw128(sV + (uint32_t)(gp % NSV) * kPairBytes, 16384, 1024);
                        const int steps = (2 * j + 1 < n_union) ? 8 : 4;
#pragma unroll
                        for (int s = 0; s < 8; ++s)
                            if (s < steps)
                                mma_f16_ts(tmem + kColO, pa + 8u * s, dv + (uint64_t)((2048u * s) >> 4), idesc_pv,
                                           (j > 0 || s > 0) ? 1u : 0u);
                        mma_commit(BAR(BR::PV_DONE + (gp & 1)));
                    }
                }
                if (ok && !keys) mma_commit(BAR(BR::O_FULL));
                gp0 += n_pairs;
            }
            // drain: every MMA this thread issued completes before TMEM is released
            const uint32_t done = BAR(BR::MMA_DONE + (keys ? 0 : 1));
            mma_commit(done);
            mbar_drain(done, 0, kDrainNs);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps: bookkeeping between tiles, softmax, epilogue ----------
        const int stid = tid - 128;   // 0 .. 383
        const int grp = (warp - 4) >> 2;
        const int qq = warp & 3;
        const int r = 32 * qq + lane, h = r % G, qi = r / G;
        const float sl2 = p.scale * 1.4426950408889634f;
        const uint32_t lane_off = (uint32_t)(32 * qq) << 16;

        // the selection rows of tile tau into selbuf / scbuf: plain loads (sync = true) or asynchronous
        // copies waited for before the next build
        auto load_rows = [&](int tau, bool sync) {
            const TileId T = tile_of(tau, tiles_x, p, BQ);
            const int32_t *sel_base = sel_idx + ((((size_t)T.b * p.Hkv + T.g) * p.N) + T.q0) * p.k;
            for (int e = stid; e < T.nq * p.k; e += kSM) {
                if (sync) selbuf[e] = __ldg(sel_base + e);
                else cp_async4(selbuf + e, sel_base + e);
            }
            for (int e = stid; e < G * T.nq * ns; e += kSM) {
                const int hh = e / (T.nq * ns), rem = e % (T.nq * ns);
                const size_t row0 = (((size_t)T.b * p.H + (size_t)T.g * G + hh) * p.N) + T.q0;
                float *dst = scbuf + ((rem / ns) * G + hh) * ns + rem % ns;
                if (sync) *dst = __ldg(sel_score + row0 * ns + rem);
                else cp_async4(dst, sel_score + row0 * ns + rem);
            }
            if (!sync) cp_async_commit();
        };

        // the chunk union (ascending), per-query chunk lists and per-row fusion weights of tile tau,
        // from selbuf / scbuf (complete and visible to every softmax thread on entry)
        auto build = [&](int tau, int bk) {
            const TileId T = tile_of(tau, tiles_x, p, BQ);
            int *uni = uni0 + bk * uni_step;
            for (int i2 = stid; i2 < nwords; i2 += kSM) bitmap[i2] = 0u;
            sm_sync();
            const int n_marks = T.nq * p.k + T.nq;
            for (int e0 = (warp - 4) * 32; e0 < n_marks; e0 += kSM) {
                const int e = e0 + lane;
                int c = -1;
                if (e < T.nq * p.k) c = selbuf[e];
                else if (e < n_marks) c = (int)(((long long)p.q_offset + T.q0 + (e - T.nq * p.k)) / kChunk);
                if (nwords <= 8) {
                    for (int wd = 0; wd < nwords; ++wd) {
                        const unsigned int bits =
                            __reduce_or_sync(0xFFFFFFFFu, (c >= 0 && (c >> 5) == wd) ? (1u << (c & 31)) : 0u);
                        if (lane == 0 && bits) atomicOr(&bitmap[wd], bits);
                    }
                } else if (c >= 0) {
                    atomicOr(&bitmap[c >> 5], 1u << (c & 31));
                }
            }
            sm_sync();
            if (warp == 4) {
                int running = 0;
                for (int w0 = 0; w0 < nwords; w0 += 32) {
                    uint32_t word = (w0 + lane < nwords) ? bitmap[w0 + lane] : 0u;
                    const int cnt = __popc(word);
                    int incl = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    int off = running + incl - cnt;
                    while (word) {
                        const int bit = __ffs(word) - 1;
                        uni[off++] = (w0 + lane) * 32 + bit;
                        word &= word - 1;
                    }
                    running += __shfl_sync(0xFFFFFFFFu, incl, 31);
                }
                if (lane == 0) n_union_s[bk] = running;
            } else {
                for (int e = stid - 32; e < T.nq * ns; e += kSM - 32) {
                    const int q = e / ns, j = e % ns;
                    const int own_c = (int)(((long long)p.q_offset + T.q0 + q) / kChunk);
                    const int *sl = selbuf + q * p.k;
                    const int c = (j < p.k) ? sl[j] : own_c;
                    if (c < 0) continue;
                    int rank = 0;
                    for (int j2 = 0; j2 < p.k; ++j2) rank += (unsigned)sl[j2] < (unsigned)c;   // -1 never counts
                    rank += own_c < c;
                    qlist[q * ns + rank] = c;
                    qslot[q * ns + rank] = j;
                    if (j == p.k) qcnt[q] = rank + 1;   // the own chunk is the largest
                }
            }
            sm_sync();
            if (stid < kRows) {   // fusion weights, in the order of each query's chunk list
                const int rr = stid, q = rr / G;
                if (q < T.nq) {
                    const float *sc = scbuf + rr * ns;
                    float M = -INFINITY;
                    for (int j = 0; j < ns; ++j) M = fmaxf(M, sc[j]);
                    float Z = 0.f;
                    for (int j = 0; j < ns; ++j) Z += (sc[j] == -INFINITY) ? 0.f : __expf(sc[j] - M);
                    const float iz = 1.0f / Z;
                    const int *slt = qslot + q * ns;
                    const int cnt = qcnt[q];
                    for (int pos = 0; pos < cnt; ++pos) {
                        const float sj = sc[slt[pos]];
                        wts[rr * ns + pos] = (sj == -INFINITY) ? 0.f : __expf(sj - M) * iz;
                    }
                }
            }
            sm_sync();
            if (stid == 0) mbar_arrive(BAR(BR::BOOK + bk));
        };

        int tau = (int)blockIdx.x;
        if (tau < n_tiles) {
            load_rows(tau, true);
            sm_sync();
            build(tau, 0);
            if (tau + stride < n_tiles) load_rows(tau + stride, false);
        }

        int pg = 0;
        bool ok = true;
        for (int i = 0; tau < n_tiles; ++i, tau += stride) {
            const int bk = i & 1;
            const int n_union = n_union_s[bk];
            // the row's position and chunk list (positions fit in int: the ABI takes int sizes)
            const int q0 = (tiles_x - 1 - tau % tiles_x) * BQ;
            const int pos = p.q_offset + q0 + qi;
            const bool wide = __ldg(wide_flags + tau / tiles_x) != 0u;   // tau / tiles_x = b * Hkv + g
            const int own = pos / kChunk;
            const int cnt = qi < min(BQ, p.N - q0) ? qcnt[qi] : 0;
            const int lbase = qi * ns, wbase = r * ns;
            int ptr = 0;
            for (int t = grp; ok && t < n_union; t += kGroups) {
                const int gp = pg + (t >> 1), sb = gp & 1, pb = gp & 1;
                const uint32_t arrivals = (t == n_union - 1 && (n_union & 1)) ? 2u : 1u;   // a lone chunk counts twice
                if (!warp_wait(BAR(BR::QK_DONE + sb), (uint32_t)((gp >> 1) & 1), limit_ns, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t sv[64];
                const uint32_t tS = tmem + lane_off + (uint32_t)sb * 128u + (uint32_t)(t & 1) * 64u;
                tmem_ld32(tS, sv);
                tmem_ld32(tS + 32u, sv + 32);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_n(BAR(BR::QK_READY + sb), arrivals);

                const int c = uni0[bk * uni_step + t];
                while (ptr < cnt && qlist[lbase + ptr] < c) ++ptr;
                const float w = (ptr < cnt && qlist[lbase + ptr] == c) ? wts[wbase + ptr] : 0.f;
                uint32_t pk[32];
                if (__any_sync(0xFFFFFFFFu, w > 0.f)) {
                    const int n_vis = (c == own) ? pos - c * kChunk + 1 : kChunk;
                    chunk_softmax_row<kPolyPairEvery>(sv, n_vis, w, sl2, pk, wide);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = 0u;
                }
                if (gp >= kPB &&
                    !warp_wait(BAR(BR::PV_DONE + pb), (uint32_t)(((gp >> 1) - 1) & 1), limit_ns, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tmem_st32(tmem + lane_off + kColP + (uint32_t)pb * 64u + (uint32_t)(t & 1) * 32u, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_n(BAR(BR::PV_READY + pb), arrivals);
            }
            pg += (n_union + 1) >> 1;
            const bool has_next = tau + stride < n_tiles;
            // every softmax warp is past the tile's chunks: the bookkeeping may be rebuilt
            if (sm_sync_any(!ok)) {
                ok = false;
                break;
            }
            if (has_next) {
                cp_async_wait_all();
                sm_sync();
                build(tau + stride, bk ^ 1);
                if (tau + 2 * stride < n_tiles) load_rows(tau + 2 * stride, false);
            }
            // epilogue of this tile (the next tile's first products run meanwhile)
            if (warp_wait(BAR(BR::O_FULL), (uint32_t)(i & 1), limit_ns, abort_flag, status)) {
                tc_fence_after();
                const TileId T = tile_of(tau, tiles_x, p, BQ);
                const bool valid = qi < T.nq;
                Tout *orow = O + ((((size_t)T.b * p.H + (size_t)T.g * G + h) * p.N) + T.q0 + qi) * kD;
                for (int cb = grp; cb < kD / 32; cb += kGroups) {
                    const int col = cb * 32;
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_off + kColO + (uint32_t)col, v);
                    tmem_wait_ld();
                    if (valid) store_row32(orow + col, v);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(BAR(BR::O_EMPTY));
            } else {
                ok = false;
            }
        }
        cp_async_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The driver's tensor-map encoder, looked up through the runtime so that the
// library itself does not link against libcuda (it loads on machines without a
// GPU driver; the lookup happens on the first launch).
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

bool encode(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, int rank, const cuuint64_t *dims,
            const cuuint64_t *strides, const cuuint32_t *box)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(ptr),
                                        dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int kSmemLimit = 227 * 1024;

// Deepest value ring that fits (the key ring always has kSP pair slots): 0 = 2 value pair slots,
// 1 = 1, -1 = none.
int ring_config(int k, int nwords, int BQ)
{
    if (make_layout(kSP, 2, k, nwords, BQ).total + 1024 <= kSmemLimit) return 0;
    if (make_layout(kSP, 1, k, nwords, BQ).total + 1024 <= kSmemLimit) return 1;
    return -1;
}

template <int G, typename Tout>
cudaError_t launch_g(const Dims &p, const void *Q, const void *K, const void *V16, const void *V,
                     const unsigned int *wide_flags, const int32_t *sel_idx, const float *sel_score, void *O,
                     const DeviceCtl &ctl, cudaStream_t s)
{
    constexpr int BQ = kRows / G;
    CUtensorMap tq, tk, tv, tvb;
    // Q viewed as (d, head, query): a box of G heads x BQ queries lands query-major, row = query * G + head
    const cuuint64_t qd[3] = {(cuuint64_t)kD, (cuuint64_t)p.B * p.H, (cuuint64_t)p.N};
    const cuuint64_t qs[2] = {(cuuint64_t)p.N * kD * 2, (cuuint64_t)kD * 2};
    const cuuint32_t qb[3] = {64, (cuuint32_t)G, (cuuint32_t)BQ};
    const cuuint64_t kd[2] = {(cuuint64_t)kD, (cuuint64_t)p.B * p.Hkv * p.T};
    const cuuint64_t ks[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t kb[2] = {64, (cuuint32_t)kChunk};
    if (!encode(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, 3, qd, qs, qb) ||
        !encode(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, 2, kd, ks, kb) ||
        !encode(&tv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, V16, 2, kd, ks, kb) ||
        !encode(&tvb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 2, kd, ks, kb))
        return cudaErrorInvalidValue;
    const int c_max = (int)(((long long)p.q_offset + p.N - 1) / kChunk);
    const int nwords = c_max / 32 + 1;
    const int tiles_x = (p.N + BQ - 1) / BQ;
    const int n_tiles = tiles_x * p.Hkv * p.B;
    static int n_sm = 0;
    if (n_sm == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm < 1)
            return cudaErrorInvalidValue;
    }
    dim3 grid((unsigned)(n_tiles < n_sm ? n_tiles : n_sm));
    const int cfg = ring_config(p.k, nwords, BQ);
    cudaError_t e = cudaErrorInvalidValue;
#define HILS_LAUNCH_TC(NV)                                                                                  \
    {                                                                                                        \
        const size_t smem = make_layout(kSP, NV, p.k, nwords, BQ).total + 1024;                             \
        auto kern = attend_tc_persistent_kernel<G, Tout, NV>;                                                          \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);              \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, kThreads, smem, s>>>(tq, tk, tv, tvb, p, sel_idx, sel_score, wide_flags,                 \
                                          static_cast<Tout *>(O),                                            \
                                          ctl.status, (unsigned long long)ctl.wait_limit, nwords,            \
                                          ctl.inject_stall, n_tiles, tiles_x);                               \
    }
    if (cfg == 0) HILS_LAUNCH_TC(2)
    else HILS_LAUNCH_TC(1)
#undef HILS_LAUNCH_TC
    return cudaGetLastError();
}

template <typename Tout>
cudaError_t launch_o(const Dims &p, const void *Q, const void *K, const void *V16, const void *V,
                     const unsigned int *wide, const int32_t *sel_idx, const float *sel_score, void *O,
                     const DeviceCtl &ctl, cudaStream_t s)
{
    switch (p.G) {
    case 1: return launch_g<1, Tout>(p, Q, K, V16, V, wide, sel_idx, sel_score, O, ctl, s);
    case 2: return launch_g<2, Tout>(p, Q, K, V16, V, wide, sel_idx, sel_score, O, ctl, s);
    case 4: return launch_g<4, Tout>(p, Q, K, V16, V, wide, sel_idx, sel_score, O, ctl, s);
    case 8: return launch_g<8, Tout>(p, Q, K, V16, V, wide, sel_idx, sel_score, O, ctl, s);
    default: return launch_g<16, Tout>(p, Q, K, V16, V, wide, sel_idx, sel_score, O, ctl, s);
    }
}

}  // namespace

// Whether the tensor-core kernel covers this problem.
bool attend_tc_persistent_supported(const Dims &p, hils_dtype in)
{
    if (in != HILS_BF16 || p.d != kD || p.C != kChunk || p.N < 2) return false;
    if (p.G != 1 && p.G != 2 && p.G != 4 && p.G != 8 && p.G != 16) return false;
    const int c_max = (int)(((long long)p.q_offset + p.N - 1) / kChunk);
    return ring_config(p.k, c_max / 32 + 1, kRows / p.G) >= 0;
}

cudaError_t launch_attend_prefill_tc_persistent(const Dims &p, hils_dtype out, const void *Q, const void *K,
                                                const void *V, const int32_t *sel_idx, const float *sel_score,
                                                void *O, void *ws, const DeviceCtl &ctl, cudaStream_t s)
{
    cudaError_t e = launch_v_to_f16(p, V, ws, s);
    if (e != cudaSuccess) return e;
    const unsigned int *wide = attend_tc_wide_flags(p, ws);
    if (out == HILS_F32) return launch_o<float>(p, Q, K, ws, V, wide, sel_idx, sel_score, O, ctl, s);
    return launch_o<__nv_bfloat16>(p, Q, K, ws, V, wide, sel_idx, sel_score, O, ctl, s);
}

}  // namespace hils
