// attend_prefill_tc.cu -- chunk attention and fusion on the sm_100a tensor cores (bf16 in, d = 128, C = 64).
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
// Value product precision.  The definition holds for any finite input, and V
// enters the product exactly in both of two forms.  A streaming pass converts V
// to f16 once per call and flags every (b, kv-head) slice holding a value of
// magnitude >= 65536, where f16 overflows (every bf16 value below that is
// exact in f16; the few below 2^-14 become f16 subnormals, within 2^-25).  A
// block of an unflagged slice reads the f16 copy and rounds P to f16 (relative
// 2^-11); a block of a flagged slice reads V as given and rounds P to bf16
// (relative 2^-8).  The output error from rounding P is at most that relative
// error times the largest |v| the row attends to (the row's P sums to one).
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
    uint32_t q, k, v, bar, misc, bitmap, uni, selbuf, scbuf, qlist, qslot, qcnt, wts, total;
};

__host__ __device__ inline uint32_t al16(uint32_t x) { return (x + 15u) & ~15u; }

constexpr int kMaxBars = 64;

// Shared memory: Q (32 KB), kSP key slots and NSV value slots (two chunks, 32 KB each), barriers,
// then the block's selection bookkeeping.
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
    L.uni = al16(L.bitmap + 4u * (uint32_t)nwords);
    L.selbuf = al16(L.uni + 4u * ns * (uint32_t)BQ);               // the block's sel_idx rows
    L.scbuf = al16(L.selbuf + 4u * (uint32_t)k * (uint32_t)BQ);    // the rows' sel_score values
    L.qlist = al16(L.scbuf + 4u * ns * (uint32_t)kRows);
    L.qslot = al16(L.qlist + 4u * ns * (uint32_t)BQ);
    L.qcnt = al16(L.qslot + 4u * ns * (uint32_t)BQ);
    L.wts = al16(L.qcnt + 4u * (uint32_t)BQ);
    L.total = al16(L.wts + 4u * ns * (uint32_t)kRows);
    return L;
}

// Barrier slots.  Key slot / S buffer b (pair p uses b = p % 2), P buffer b (p % 2 as well: TMEM
// always holds two) and value slot v (p % NSV):
//   K_LAND[b]    the pair's key tiles have landed (TMA transaction count)
//   QK_READY[b]  S buffer b may take pair p: its key tiles are in (the key loader's arrival) and all
//                eight softmax warps of its two chunks have read pair p - 2 out of it
//   QK_DONE[b]   the key product of pair p is complete: S is ready and the key slot is free
//   V_LAND[v]    the pair's value tiles have landed
//   PV_READY[b]  the value product of pair p may start: its values are in (the value loader's
//                arrival) and the eight softmax warps of its two chunks wrote P buffer b
//   PV_DONE[b]   the value product of pair p is complete: P buffer b is free, and so is the value
//                slot of pair p
// so the MMA issuer tests one barrier per product and commits to one.  P buffers and their barriers
// go by p % 2 even with a single value slot: a softmax warp skips pairs (chunk t goes to group
// t % 3), and a parity wait is only sound while the waiter is at most one phase behind, which two
// P buffers guarantee (a warp that writes pair p has already seen the value product of p - 4 done)
// and one would not.
template <int NSV>
struct Bars {
    static constexpr int Q_FULL = 0, K_LAND = 1, QK_READY = K_LAND + kSP, QK_DONE = QK_READY + kSP,
                         V_LAND = QK_DONE + kSP, PV_READY = V_LAND + NSV, PV_DONE = PV_READY + kPB,
                         O_FULL = PV_DONE + kPB, MMA_DONE = O_FULL + 1;   // MMA_DONE + 0/1: the two issuers
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

// One loader thread streams n tiles through a ring of `slots` buffers: tile i goes to slot i % slots
// once the consumer has finished tile i - slots (completion barriers `done` go by tile % 2), lands on
// `land` (by slot), and is then announced on `ready` (by tile % 2; other arrivals may share it; the
// last tile's announcement counts 1 + tail_extra arrivals).  Up to `slots` tiles are in flight.  On
// an abort the thread waits, with its own bound, for the copies it started.  Returns the tiles
// announced.
template <typename Issue>
__device__ __forceinline__ int stream_tiles(int n, int slots, uint32_t done0, uint32_t land0, uint32_t ready0,
                                            Issue &&issue, int tail_extra, unsigned long long limit_ns,
                                            volatile int *abort_flag, unsigned int *status)
{
    int issued = 0, landed = 0;
    long long t_prog = cycle_now();
    bool ok = true;
    while (landed < n) {
        const int freed = issued - slots;   // the tile that last used the next slot
        if (issued < n && issued < landed + slots &&
            (freed < 0 || mbar_test(done0 + 8u * (uint32_t)(freed & 1), (uint32_t)((freed >> 1) & 1)))) {
            issue(issued);
            ++issued;
            t_prog = cycle_now();
            continue;
        }
        const uint32_t lbar = land0 + 8u * (uint32_t)(landed % slots);
        const uint32_t lphase = (uint32_t)((landed / slots) & 1);
        if (landed < issued && mbar_test(lbar, lphase)) {
            const int n_arrive = (landed == n - 1) ? 1 + tail_extra : 1;
            for (int a = 0; a < n_arrive; ++a) mbar_arrive(ready0 + 8u * (uint32_t)(landed & 1));
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
        for (int v = landed; v < issued; ++v)
            mbar_drain(land0 + 8u * (uint32_t)(v % slots), (uint32_t)((v / slots) & 1), kDrainNs);
    return landed;
}

template <int G, typename Tout, int NSV>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVb, Dims p,
                     const int32_t *__restrict__ sel_idx, const float *__restrict__ sel_score,
                     const unsigned int *__restrict__ wide_flags, Tout *__restrict__ O, unsigned int *status,
                     unsigned long long limit_ns, int nwords, int inject_stall)
{
    constexpr int BQ = kRows / G;
    using BR = Bars<NSV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const Layout Ly = make_layout(kSP, NSV, p.k, nwords, BQ);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // later query tiles select from more chunks and take longer: they are dispatched first, so that
    // the grid ends on short blocks
    const int q0 = (int)(gridDim.x - 1 - blockIdx.x) * BQ, g = blockIdx.y, b = blockIdx.z;
    const int nq = min(BQ, p.N - q0);
    const int ns = p.k + 1;
    // a slice whose values overflow f16 takes the bf16 value product (V as given, P in bf16)
    const bool wide = __ldg(wide_flags + b * p.Hkv + g) != 0u;
    const CUtensorMap *tmVsel = wide ? &tmVb : &tmV;

    const uint32_t sQ = smem_addr(base + Ly.q), sK = smem_addr(base + Ly.k), sV = smem_addr(base + Ly.v);
    const uint32_t bar0 = smem_addr(base + Ly.bar);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + Ly.misc);
    int *n_union_p = reinterpret_cast<int *>(base + Ly.misc + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + Ly.misc + 8);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(base + Ly.bitmap);
    int *uni = reinterpret_cast<int *>(base + Ly.uni);
    int *selbuf = reinterpret_cast<int *>(base + Ly.selbuf);
    float *scbuf = reinterpret_cast<float *>(base + Ly.scbuf);
    int *qlist = reinterpret_cast<int *>(base + Ly.qlist);
    int *qslot = reinterpret_cast<int *>(base + Ly.qslot);
    int *qcnt = reinterpret_cast<int *>(base + Ly.qcnt);
    float *wts = reinterpret_cast<float *>(base + Ly.wts);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };

    // ---- set-up --------------------------------------------------------------
    // Q's load starts at once; the selection rows are copied to shared memory with
    // coalesced loads, and the block's chunk union, per-query chunk lists and per-row
    // fusion weights are built from there.
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
        mbar_init(BAR(BR::MMA_DONE), 1);
        mbar_init(BAR(BR::MMA_DONE + 1), 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(tmVsel);
        mbar_arrive_expect_tx(BAR(BR::Q_FULL), 32768u);
        tma_load_3d(sQ, &tmQ, BAR(BR::Q_FULL), 0, b * p.H + g * G, q0);
        tma_load_3d(sQ + 16384u, &tmQ, BAR(BR::Q_FULL), 64, b * p.H + g * G, q0);
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), kTmemCols);
        tmem_relinquish();
    }
    for (int i = tid; i < nwords; i += kThreads) bitmap[i] = 0u;
    const int32_t *sel_base = sel_idx + ((((size_t)b * p.Hkv + g) * p.N) + q0) * p.k;
    for (int e = tid; e < nq * p.k; e += kThreads) selbuf[e] = __ldg(sel_base + e);
    for (int e = tid; e < G * nq * ns; e += kThreads) {
        const int h = e / (nq * ns), rem = e % (nq * ns);
        const size_t row0 = (((size_t)b * p.H + (size_t)g * G + h) * p.N) + q0;
        scbuf[((rem / ns) * G + h) * ns + rem % ns] = __ldg(sel_score + row0 * ns + rem);
    }
    __syncthreads();

    // mark the selected and own chunks; with few bitmap words the bits are OR-reduced across the
    // warp first, so that the shared-memory atomics do not all land on the same words
    const int n_marks = nq * p.k + nq;
    for (int e0 = warp * 32; e0 < n_marks; e0 += kThreads) {
        const int e = e0 + lane;
        int c = -1;
        if (e < nq * p.k) c = selbuf[e];
        else if (e < n_marks) c = (int)(((long long)p.q_offset + q0 + (e - nq * p.k)) / kChunk);
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
    __syncthreads();

    if (warp == 0) {
        // ascending list of the union's chunks
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
        if (lane == 0) *n_union_p = running;
    }
    {
        // each query's chunks (selected + own) in ascending order, with the slot each came from:
        // one thread per (query, slot) counts the query's smaller chunks (chunks are distinct)
        for (int e = tid - 32; e >= 0 && e < nq * ns; e += kThreads - 32) {
            const int qi = e / ns, j = e % ns;
            const int own_c = (int)(((long long)p.q_offset + q0 + qi) / kChunk);
            const int *sl = selbuf + qi * p.k;
            const int c = (j < p.k) ? sl[j] : own_c;
            if (c < 0) continue;
            int rank = 0;
            for (int j2 = 0; j2 < p.k; ++j2) rank += (unsigned)sl[j2] < (unsigned)c;   // -1 never counts
            rank += own_c < c;
            qlist[qi * ns + rank] = c;
            qslot[qi * ns + rank] = j;
            if (j == p.k) qcnt[qi] = rank + 1;   // the own chunk is the largest
        }
    }
    // the union and the chunk lists are complete: the loaders start now, while the first softmax
    // warps compute the fusion weights
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int n_union = *n_union_p;

    const int kv_row0 = (b * p.Hkv + g) * p.T;
    if (warp == 0) {
        // ---------------- key tiles, two chunks per slot; a slot frees when its key product completes
        if (lane == 0) {
            const int n_pairs = (n_union + 1) >> 1;
            auto issue = [&](int pr) {
                const int st = pr % kSP;
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
            const int landed = stream_tiles(n_pairs, kSP, BAR(BR::QK_DONE), BAR(BR::K_LAND), BAR(BR::QK_READY), issue,
                                            0, limit_ns, abort_flag, status);
            (void)landed;
            mbar_drain(BAR(BR::Q_FULL), 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- value tiles, two chunks per slot; a slot frees when its value product completes
        if (lane == 0) {
            const int n_pairs = (n_union + 1) >> 1;
            auto issue = [&](int pr) {
                const int st = pr % NSV;
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
            // a lone last chunk has no second softmax group to announce its P: the loader stands in
            stream_tiles(n_pairs, NSV, BAR(BR::PV_DONE), BAR(BR::V_LAND), BAR(BR::PV_READY), issue, (n_union & 1) ? 4 : 0,
                         limit_ns, abort_flag, status);
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3) {
        // ---------------- MMA issue: warp 2 the key products, warp 3 the value products ---------
        // The tensor core accepts one MMA at a time from a thread (the issue returns about when the
        // previous one is done), so each issuer's waits and bookkeeping between products would
        // leave it idle; with two issuers the other one's MMAs fill those gaps.
        if (lane == 0) {
            const bool keys = (warp == 2);
            const int n_pairs = (n_union + 1) >> 1;
            const uint32_t idesc_pv = wide ? IDESC_PV_BF16 : IDESC_PV;
            bool ok = true;
            if (keys && inject_stall) {
                // test control: wait once on a barrier nothing signals, so the bounded wait expires
                ok = mbar_wait(BAR(BR::MMA_DONE), 0, limit_ns, abort_flag, status);
            }
            if (keys) ok = ok && mbar_wait(BAR(BR::Q_FULL), 0, limit_ns, abort_flag, status);
            // descriptors of Q's eight K-steps
            uint64_t dq[8];
#pragma unroll
            for (int s = 0; s < 8; ++s) dq[s] = smem_desc_sw128(sQ + (s >> 2) * 16384u + (s & 3) * 32u, 16, 1024);
            for (int i = 0; ok && i < n_pairs; ++i) {
                const uint32_t bar = keys ? BAR(BR::QK_READY + i % kSP) : BAR(BR::PV_READY + i % kPB);
                const uint32_t phase = (uint32_t)((keys ? i / kSP : i / kPB) & 1);
                // bounded poll (a test takes ~100 cycles, so the loop costs few issue slots); the grid's
                // status word is read only now and then
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
                    const uint32_t d_s = tmem + (uint32_t)(i % kSP) * 128u;
                    const uint64_t dk = smem_desc_sw128(sK + (uint32_t)(i % kSP) * kPairBytes, 16, 1024);
                    const uint32_t idesc = (2 * i + 1 < n_union) ? IDESC_QK2 : IDESC_QK1;
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        mma_bf16_ss(d_s, dq[s], dk + (uint64_t)(((s >> 2) * 16384u + (s & 3) * 32u) >> 4), idesc,
                                    s > 0 ? 1u : 0u);
                    mma_commit(BAR(BR::QK_DONE + i % kSP));
                } else {
                    const uint32_t pa = tmem + kColP + (uint32_t)(i % kPB) * 64u;
                    const uint64_t dv = smem_desc_sw128(sV + (uint32_t)(i % NSV) * kPairBytes, 16384, 1024);
                    const int steps = (2 * i + 1 < n_union) ? 8 : 4;
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        if (s < steps)
                            mma_f16_ts(tmem + kColO, pa + 8u * s, dv + (uint64_t)((2048u * s) >> 4), idesc_pv,
                                       (i > 0 || s > 0) ? 1u : 0u);
                    mma_commit(BAR(BR::PV_DONE + i % kPB));
                }
            }
            if (ok && !keys) mma_commit(BAR(BR::O_FULL));
            // drain: every MMA this thread issued completes before TMEM is released
            const uint32_t done = BAR(BR::MMA_DONE + (keys ? 0 : 1));
            mma_commit(done);
            mbar_drain(done, 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- softmax (kGroups groups, chunks round-robin) and epilogue ----
        if (warp < 8) {
            // fusion weights of each row, in the order of its query's chunk list (warps 4..7)
            const int r = tid - 128, qi = r / G;
            if (qi < nq) {
                const float *sc = scbuf + r * ns;
                float M = -INFINITY;
                for (int j = 0; j < ns; ++j) M = fmaxf(M, sc[j]);
                float Z = 0.f;
                for (int j = 0; j < ns; ++j) Z += (sc[j] == -INFINITY) ? 0.f : __expf(sc[j] - M);
                const float iz = 1.0f / Z;
                const int *slt = qslot + qi * ns;
                const int cnt = qcnt[qi];
                for (int pos = 0; pos < cnt; ++pos) {
                    const float sj = sc[slt[pos]];
                    wts[r * ns + pos] = (sj == -INFINITY) ? 0.f : __expf(sj - M) * iz;
                }
            }
        }
        // the softmax warps wait for the weights (named barrier 1: warps 4..15 only)
        asm volatile("bar.sync 1, %0;" ::"r"(32 * 4 * kGroups) : "memory");
        const int grp = (warp - 4) >> 2;
        const int qq = warp & 3;
        const int r = 32 * qq + lane, h = r % G, qi = r / G;
        const bool valid = qi < nq;
        const long long pos = (long long)p.q_offset + q0 + qi;
        const int own = (int)(pos / kChunk);
        const int cnt = valid ? qcnt[qi] : 0;
        const int *lst = qlist + qi * ns;
        const float *wr = wts + r * ns;
        const float sl2 = p.scale * 1.4426950408889634f;
        const uint32_t lane_off = (uint32_t)(32 * qq) << 16;
        int ptr = 0;
        bool ok = true;
        for (int t = grp; t < n_union; t += kGroups) {
            const int pr = t >> 1, sb = pr % kSP, pb = pr % kPB;
            if (!warp_wait(BAR(BR::QK_DONE + sb), (uint32_t)((pr / kSP) & 1), limit_ns, abort_flag, status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sv[64];
            const uint32_t tS = tmem + lane_off + (uint32_t)sb * 128u + (uint32_t)(t & 1) * 64u;
            tmem_ld32(tS, sv);
            tmem_ld32(tS + 32u, sv + 32);
            tmem_wait_ld();
            // the scores are in registers: the S buffer may take the pair after next
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(BR::QK_READY + sb));

            const int c = uni[t];
            while (ptr < cnt && lst[ptr] < c) ++ptr;
            const float w = (ptr < cnt && lst[ptr] == c) ? wr[ptr] : 0.f;
            uint32_t pk[32];
            if (__any_sync(0xFFFFFFFFu, w > 0.f)) {   // rows with w = 0 get P = 0 from the scaling
                const int n_vis = (c == own) ? (int)(pos - (long long)c * kChunk + 1) : kChunk;
                chunk_softmax_row<kPolyPairEvery>(sv, n_vis, w, sl2, pk, wide);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) pk[j] = 0u;
            }
            if (pr >= kPB &&
                !warp_wait(BAR(BR::PV_DONE + pb), (uint32_t)(((pr / kPB) - 1) & 1), limit_ns, abort_flag, status)) {
                ok = false;
                break;
            }
            tmem_st32(tmem + lane_off + kColP + (uint32_t)pb * 64u + (uint32_t)(t & 1) * 32u, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(BR::PV_READY + pb));
        }
        if (ok && warp_wait(BAR(BR::O_FULL), 0, limit_ns, abort_flag, status)) {
            tc_fence_after();
            Tout *orow = O + ((((size_t)b * p.H + (size_t)g * G + h) * p.N) + q0 + qi) * kD;
            for (int cb = grp; cb < kD / 32; cb += kGroups) {
                const int col = cb * 32;
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + kColO + (uint32_t)col, v);
                tmem_wait_ld();
                if (valid) store_row32(orow + col, v);
            }
        }
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

// V (bf16) -> f16, 8 elements per 16-byte vector.  Every bf16 value of magnitude below 65536 is
// exact in f16 (below 2^-14 as an f16 subnormal, within 2^-25); a vector holding a larger one
// raises the flag of its (b, kv-head) slice (vec_per_slice vectors each), and the attention blocks
// of a flagged slice read V as given instead of this copy.  The flags start at zero.
__global__ void v_to_f16_kernel(const uint4 *__restrict__ in, uint4 *__restrict__ out, size_t n,
                                size_t vec_per_slice, unsigned int *__restrict__ wide_flags)
{
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const uint4 u = __ldg(in + i);
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
        bool big = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // bf16 magnitude bits >= 0x4780 means |v| >= 2^16 (or not finite)
            big |= (w[e] & 0x7FFFu) >= 0x4780u || ((w[e] >> 16) & 0x7FFFu) >= 0x4780u;
            __half2 h2 = __floats2half2_rn(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
            w[e] = *reinterpret_cast<uint32_t *>(&h2);
        }
        out[i] = make_uint4(w[0], w[1], w[2], w[3]);
        if (big) atomicOr(wide_flags + i / vec_per_slice, 1u);
    }
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
    dim3 grid((p.N + BQ - 1) / BQ, p.Hkv, p.B);
    const int cfg = ring_config(p.k, nwords, BQ);
    cudaError_t e = cudaErrorInvalidValue;
#define HILS_LAUNCH_TC(NV)                                                                                  \
    {                                                                                                        \
        const size_t smem = make_layout(kSP, NV, p.k, nwords, BQ).total + 1024;                             \
        auto kern = attend_tc_kernel<G, Tout, NV>;                                                          \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);              \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, kThreads, smem, s>>>(tq, tk, tv, tvb, p, sel_idx, sel_score, wide_flags,                 \
                                          static_cast<Tout *>(O),                                            \
                                          ctl.status, (unsigned long long)ctl.wait_limit, nwords,            \
                                          ctl.inject_stall);                                                 \
    }
    if (cfg == 0) HILS_LAUNCH_TC(2)
    else HILS_LAUNCH_TC(1)
#undef HILS_LAUNCH_TC
    return cudaGetLastError();
}

template <typename Tout>
cudaError_t launch_o(const Dims &p, const void *Q, const void *K, const void *V16, const void *V,
                     const unsigned int *wf, const int32_t *sel_idx, const float *sel_score, void *O,
                     const DeviceCtl &ctl, cudaStream_t s)
{
    switch (p.G) {
    case 1: return launch_g<1, Tout>(p, Q, K, V16, V, wf, sel_idx, sel_score, O, ctl, s);
    case 2: return launch_g<2, Tout>(p, Q, K, V16, V, wf, sel_idx, sel_score, O, ctl, s);
    case 4: return launch_g<4, Tout>(p, Q, K, V16, V, wf, sel_idx, sel_score, O, ctl, s);
    case 8: return launch_g<8, Tout>(p, Q, K, V16, V, wf, sel_idx, sel_score, O, ctl, s);
    default: return launch_g<16, Tout>(p, Q, K, V16, V, wf, sel_idx, sel_score, O, ctl, s);
    }
}

size_t v16_bytes(const Dims &p) { return align_up((size_t)p.B * p.Hkv * p.T * kD * 2, 256); }

}  // namespace

// Whether the tensor-core kernel covers this problem.
bool attend_tc_supported(const Dims &p, hils_dtype in)
{
    if (in != HILS_BF16 || p.d != kD || p.C != kChunk || p.N < 2) return false;
    if (p.G != 1 && p.G != 2 && p.G != 4 && p.G != 8 && p.G != 16) return false;
    const int c_max = (int)(((long long)p.q_offset + p.N - 1) / kChunk);
    return ring_config(p.k, c_max / 32 + 1, kRows / p.G) >= 0;
}

// V as f16, then one flag word per (b, kv-head) slice
size_t attend_tc_ws_bytes(const Dims &p)
{
    return v16_bytes(p) + align_up((size_t)p.B * p.Hkv * sizeof(unsigned int), 256);
}

// V converted to f16 into the workspace (the first v16_bytes), and one flag per (b, kv-head) slice
// that holds a value f16 cannot represent (the next B * Hkv words); the flags are cleared first.
const unsigned int *attend_tc_wide_flags(const Dims &p, const void *ws)
{
    return reinterpret_cast<const unsigned int *>(static_cast<const char *>(ws) + v16_bytes(p));
}

cudaError_t launch_v_to_f16(const Dims &p, const void *V, void *ws, cudaStream_t s)
{
    const size_t n16 = (size_t)p.B * p.Hkv * p.T * kD / 8;
    unsigned int *wide = reinterpret_cast<unsigned int *>(static_cast<char *>(ws) + v16_bytes(p));
    cudaError_t e = cudaMemsetAsync(wide, 0, (size_t)p.B * p.Hkv * sizeof(unsigned int), s);
    if (e != cudaSuccess) return e;
    v_to_f16_kernel<<<148 * 8, 256, 0, s>>>(static_cast<const uint4 *>(V), static_cast<uint4 *>(ws), n16,
                                            (size_t)p.T * kD / 8, wide);
    return cudaGetLastError();
}

cudaError_t launch_attend_prefill_tc(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                     const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                     const DeviceCtl &ctl, cudaStream_t s)
{
    cudaError_t e = launch_v_to_f16(p, V, ws, s);
    if (e != cudaSuccess) return e;
    unsigned int *wide = reinterpret_cast<unsigned int *>(static_cast<char *>(ws) + v16_bytes(p));
    if (out == HILS_F32) return launch_o<float>(p, Q, K, ws, V, wide, sel_idx, sel_score, O, ctl, s);
    return launch_o<__nv_bfloat16>(p, Q, K, ws, V, wide, sel_idx, sel_score, O, ctl, s);
}

}  // namespace hils
