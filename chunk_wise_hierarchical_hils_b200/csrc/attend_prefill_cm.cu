// attend_prefill_cm.cu -- chunk attention and fusion for prefill, chunk-major, on the sm_100a tensor
// cores (bf16 in, d = 128, C = 64).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1): Abstract and Sec. 3 "Hierarchical
// softmax" (softmax inside every selected chunk; the chunk outputs fused by a softmax over the
// retrieval scores); Sec. 4 "Architecture" (a GQA group's heads share the retrieved chunks).  The
// pages' kernel idea (Sec. 4, "Kernel design") batches adjacent queries over the union of their
// chunks, which pays when adjacent queries share most of their chunks (Sec. 7, "Adjacent-query chunk
// sharing").  When they do not, a query block's union is nearly every visible chunk, and most of the
// block's rows do no useful work on most chunks.  This kernel turns the selection around instead:
// for every chunk, the query rows that selected it.
//
//   inversion  a counting sort of the selection by (kv-group, query range, chunk) gives, per chunk,
//              the list of (query, slot) entries that selected it; tiles are up to 128 / G of those
//              queries (x G heads = 128 rows), plus tiles of the queries whose own chunk it is (causal);
//   attention  a persistent kernel walks the tiles: gathers the tile's query rows (16-byte
//              asynchronous copies into the 128-byte-swizzled layout), loads the chunk's keys and values
//              (TMA), computes S = Q K^T (tcgen05, M = 128 rows, N = 64 keys) into TMEM; the softmax warps
//              write P = w_c softmax(S) (the fusion weight folded in, f16) to shared memory; then
//              O^T = V^T P^T (tcgen05, M = d = 128, N = 128 rows, K = 64 keys), so that TMEM lane x
//              holds column x of every row's chunk output; the epilogue warps copy it, half a tile at
//              a time, into the tile's query buffer (free once S is computed) as rows of d floats, and
//              one thread adds each query's G rows into a float32 accumulator [B][Hkv][N][G][d] with a
//              single bulk reduction (cp.reduce.async.bulk ... add.f32, G * d * 4 bytes, no multicast);
//   ordering   tiles go (kv-group, query range, chunk): the accumulator rows of one query range
//              (about 32 MB) stay in L2 while its tiles run, so the reductions do not reach HBM;
//   finalize   the accumulator is permuted to O [B][H][N][d] in the output type.
// Each chunk's softmax is normalised on its own and the fusion weights are known, so the partial
// outputs simply add (in no fixed order: the last bits of the float32 sums may differ between runs).
// A slice of V holding a value f16 cannot represent takes the bf16 value product (V as given).
// Every wait is bounded: on expiry the CTA records HILS_ERR_TIMEOUT, drains what it started and exits.
#include <cuda.h>
#include <cuda_fp16.h>

#include "chunk_softmax.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kD = 128, kC = 64, kRows = 128;
constexpr int kThreads = 512;              // 16 warps: roles below
constexpr uint32_t kQTile = 32768;         // 128 rows x 128 d, bf16, two 64-column halves
constexpr uint32_t kKVTile = 32768;        // keys (two halves of 8 KB), then values (two halves)
constexpr uint32_t kPTile = 16384;         // 128 rows x 64 keys, 16-bit
constexpr uint32_t kTmemCols = 512;        // S (2 x 64 columns), O^T (2 x 128 columns)
constexpr uint32_t kColO = 128;
constexpr int kPolyPairEvery = 4;
constexpr unsigned long long kDrainNs = 2000000000ull;
constexpr int kOwnBit = 0x40000000;
constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_f16_f32(128, 128, true, false);        // A = V^T (MN-major), B = P^T
constexpr uint32_t IDESC_PV_BF16 = idesc_bf16_f32(128, 128, true, false);

// shared memory (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;                               // 2 query tiles
constexpr uint32_t OFF_KV = OFF_Q + 2 * kQTile;             // 2 key/value tiles
constexpr uint32_t OFF_P = OFF_KV + 2 * kKVTile;            // 2 probability tiles
constexpr uint32_t OFF_RQ = OFF_P + 2 * kPTile;             // [2][128] int: per tile query q: its accumulator
                                                            // block (b Hkv + g) N + i, -1 = none
constexpr uint32_t OFF_RW = OFF_RQ + 2 * kRows * 4;         // [2][128] float: fusion weight
constexpr uint32_t OFF_RN = OFF_RW + 2 * kRows * 4;         // [2][128] int: visible keys
constexpr uint32_t OFF_TM = OFF_RN + 2 * kRows * 4;          // [2] int4: the tile's kv-group, chunk, -, V flag
constexpr uint32_t OFF_BAR = OFF_TM + 2 * 16;
constexpr uint32_t OFF_MISC = OFF_BAR + 32 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;

// barriers (index; each pair by tile parity)
enum {
    B_QG = 0,        // query rows of the tile landed (128 gather threads)
    B_ROW = 2,       // the tile's row information written (128 gather threads)
    B_KV = 4,        // keys and values landed (TMA transaction count)
    B_SFULL = 6,     // S computed (MMA commit)
    B_SFREE = 8,     // S read out of TMEM (4 softmax warps)
    B_PFULL = 10,    // P written (128 softmax threads)
    B_OFULL = 12,    // O^T computed (MMA commit)
    B_OFREE = 14,    // O^T read out of TMEM (4 epilogue warps)
    B_KVPFREE = 16,  // value product done: key/value tile and P tile free (MMA commit)
    B_MMADONE = 18
};

// the epilogue's four warps meet on named barrier 3; the OR of their flags says whether any stops
__device__ __forceinline__ bool epilogue_bar_any(bool flag)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 3, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(flag ? 1u : 0u)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void bulk_reduce_add_f32(float *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;"
                 ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, unsigned long long lim, volatile int *abort_flag,
                                          unsigned int *status)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, lim, abort_flag, status) ? 1 : 0;
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    attend_cm_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV16,
                     const __grid_constant__ CUtensorMap tmVb, Dims p, const __nv_bfloat16 *__restrict__ Q,
                     const float *__restrict__ ew, const float *__restrict__ ow,
                     const int *__restrict__ entries, const int4 *__restrict__ tiles, const int *__restrict__ n_tiles_p,
                     const unsigned int *__restrict__ wide_flags, float *__restrict__ acc, unsigned int *status,
                     unsigned long long limit_ns)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *base = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sQ = smem_addr(base + OFF_Q), sKV = smem_addr(base + OFF_KV), sP = smem_addr(base + OFF_P);
    int *rq = reinterpret_cast<int *>(base + OFF_RQ);
    float *rw = reinterpret_cast<float *>(base + OFF_RW);
    int *rn = reinterpret_cast<int *>(base + OFF_RN);
    int4 *tm = reinterpret_cast<int4 *>(base + OFF_TM);
    const uint32_t bar0 = smem_addr(base + OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(base + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(base + OFF_MISC + 4);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int n_tiles = __ldg(n_tiles_p);
    const int G = p.G;
    auto tile_of = [&](int t) { return (int)blockIdx.x + t * (int)gridDim.x; };

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_QG + b), 128);
            mbar_init(BAR(B_ROW + b), 128);
            mbar_init(BAR(B_KV + b), 1);
            mbar_init(BAR(B_SFULL + b), 1);
            mbar_init(BAR(B_SFREE + b), 4);
            mbar_init(BAR(B_PFULL + b), 128);
            mbar_init(BAR(B_OFULL + b), 1);
            mbar_init(BAR(B_OFREE + b), 4);
            mbar_init(BAR(B_KVPFREE + b), 1);
        }
        mbar_init(BAR(B_MMADONE), 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV16);
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
        // ---- keys and values of each tile's chunk (TMA); the tile's value product frees the buffer
        if (lane == 0) {
            int issued = 0;
            for (int t = 0; tile_of(t) < n_tiles; ++t) {
                const int b = t & 1;
                if (t >= 2 && !mbar_wait(BAR(B_KVPFREE + b), (uint32_t)(((t >> 1) - 1) & 1), limit_ns, abort_flag, status))
                    break;
                const int4 d = __ldg(tiles + tile_of(t));
                const int c = d.y & ~kOwnBit;
                const int row = d.x * p.T + c * kC;
                const CUtensorMap *tv = __ldg(wide_flags + d.x) ? &tmVb : &tmV16;
                const uint32_t dst = sKV + (uint32_t)b * kKVTile;
                mbar_arrive_expect_tx(BAR(B_KV + b), kKVTile);
                tma_load_2d(dst, &tmK, BAR(B_KV + b), 0, row);
                tma_load_2d(dst + 8192u, &tmK, BAR(B_KV + b), 64, row);
                tma_load_2d(dst + 16384u, tv, BAR(B_KV + b), 0, row);
                tma_load_2d(dst + 24576u, tv, BAR(B_KV + b), 64, row);
                ++issued;
            }
            if (*abort_flag)   // the copies started must land before the CTA exits
                for (int u = max(0, issued - 2); u < issued; ++u)
                    mbar_drain(BAR(B_KV + (u & 1)), (uint32_t)((u >> 1) & 1), kDrainNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issue: S(t + 1) = Q K^T, then O^T(t) = V^T P^T
        if (lane == 0) {
            bool ok = true;
            auto mma_qk = [&](int t) {
                const int b = t & 1;
                const uint32_t ph = (uint32_t)((t >> 1) & 1);
                if (!mbar_wait(BAR(B_QG + b), ph, limit_ns, abort_flag, status)) return false;
                if (!mbar_wait(BAR(B_KV + b), ph, limit_ns, abort_flag, status)) return false;
                if (t >= 2 && !mbar_wait(BAR(B_SFREE + b), ph ^ 1u, limit_ns, abort_flag, status)) return false;
                tc_fence_after();
                const uint32_t qa = sQ + (uint32_t)b * kQTile, ka = sKV + (uint32_t)b * kKVTile;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16_ss(tmem + (uint32_t)b * 64u,
                                smem_desc_sw128(qa + (uint32_t)(s >> 2) * 16384u + (uint32_t)(s & 3) * 32u, 16, 1024),
                                smem_desc_sw128(ka + (uint32_t)(s >> 2) * 8192u + (uint32_t)(s & 3) * 32u, 16, 1024),
                                IDESC_QK, s > 0 ? 1u : 0u);
                mma_commit(BAR(B_SFULL + b));
                return true;
            };
            auto mma_pv = [&](int t) {
                const int b = t & 1;
                const uint32_t ph = (uint32_t)((t >> 1) & 1);
                if (!mbar_wait(BAR(B_PFULL + b), ph, limit_ns, abort_flag, status)) return false;
                if (t >= 2 && !mbar_wait(BAR(B_OFREE + b), ph ^ 1u, limit_ns, abort_flag, status)) return false;
                tc_fence_after();
                const uint32_t idesc = tm[b].w ? IDESC_PV_BF16 : IDESC_PV;   // published with the rows
                const uint32_t va = sKV + (uint32_t)b * kKVTile + 16384u, pa = sP + (uint32_t)b * kPTile;
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16_ss(tmem + kColO + (uint32_t)b * 128u, smem_desc_sw128(va + 2048u * (uint32_t)s, 8192, 1024),
                                smem_desc_sw128(pa + 32u * (uint32_t)s, 16, 1024), idesc, s > 0 ? 1u : 0u);
                mma_commit(BAR(B_OFULL + b));
                mma_commit(BAR(B_KVPFREE + b));
                return true;
            };
            if (tile_of(0) < n_tiles) ok = mma_qk(0);
            for (int t = 0; ok && tile_of(t) < n_tiles; ++t) {
                if (tile_of(t + 1) < n_tiles) ok = mma_qk(t + 1);
                ok = ok && mma_pv(t);
            }
            mma_commit(BAR(B_MMADONE));
            mbar_drain(BAR(B_MMADONE), 0, kDrainNs);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ---- row gather: one thread per row (query q = r / G, head r % G) ----------------------------
        const int r = tid - 128, ql = r / G, h = r % G;
        int t = 0;
        bool ok = true;
        for (; tile_of(t) < n_tiles; ++t) {
            const int b = t & 1;
            if (t >= 1) {
                // the previous tile's copies: landed, made visible to the tensor core, announced
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                fence_proxy_async_smem();
                mbar_arrive(BAR(B_QG + ((t - 1) & 1)));
            }
            if (t >= 2 && !wait_warp(BAR(B_OFREE + b), (uint32_t)(((t >> 1) - 1) & 1), limit_ns, abort_flag, status)) {
                ok = false;
                break;
            }
            const int4 d = __ldg(tiles + tile_of(t));
            const int bg = d.x, c = d.y & ~kOwnBit, own = (d.y & kOwnBit) != 0, start = d.z, count = d.w;
            const int bb = bg / p.Hkv, g = bg % p.Hkv;
            const int hh = g * G + h;
            int i = -1;
            float wt = 0.f;
            if (ql < count) {
                if (own) {
                    i = start + ql;
                    wt = __ldg(ow + ((size_t)bb * p.H + hh) * p.N + i);
                } else {
                    // the entry and its fusion weights come from the inversion, loaded together
                    const int e = __ldg(entries + start + ql);
                    wt = __ldg(ew + (size_t)(start + ql) * G + h);
                    i = e >> 6;
                }
            }
            if (r == 0) tm[b] = make_int4(bg, c, own, (int)__ldg(wide_flags + bg));
            int row = -1, nvis = 0;
            if (i >= 0) {
                row = (bb * p.H + hh) * p.N + i;
                const long long pos = (long long)p.q_offset + i;
                nvis = own ? (int)(pos - (long long)c * kC + 1) : kC;
            }
            if (h == 0) rq[b * kRows + ql] = i >= 0 ? bg * p.N + i : -1;
            rw[b * kRows + r] = wt;
            rn[b * kRows + r] = nvis;
            mbar_arrive(BAR(B_ROW + b));
            // the row's 16 pieces, swizzled (piece j of a 64-column half at j ^ (r % 8)); a missing row is zeros
            const __nv_bfloat16 *src = Q + (size_t)(row >= 0 ? row : 0) * kD;
            const uint32_t sz = row >= 0 ? 16u : 0u;
            const uint32_t dst0 = sQ + (uint32_t)b * kQTile + (uint32_t)r * 128u;
#pragma unroll
            for (int pc = 0; pc < 16; ++pc) {
                const uint32_t dst = dst0 + (uint32_t)(pc >> 3) * 16384u + (uint32_t)(((pc & 7) ^ (r & 7)) << 4);
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src + pc * 8), "r"(sz)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        if (ok && t >= 1) {
            fence_proxy_async_smem();
            mbar_arrive(BAR(B_QG + ((t - 1) & 1)));
        }
    } else if (warp >= 8 && warp < 12) {
        // ---- softmax: one thread per row; P = w * softmax(S) over the visible keys -------------------
        const int r = tid - 256;
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const float sl2 = p.scale * 1.4426950408889634f;
        for (int t = 0; tile_of(t) < n_tiles; ++t) {
            const int b = t & 1;
            const uint32_t ph = (uint32_t)((t >> 1) & 1);
            if (!wait_warp(BAR(B_ROW + b), ph, limit_ns, abort_flag, status)) break;
            if (!wait_warp(BAR(B_SFULL + b), ph, limit_ns, abort_flag, status)) break;
            tc_fence_after();
            uint32_t sv[64];
            tmem_ld32(tmem + lane_off + (uint32_t)b * 64u, sv);
            tmem_ld32(tmem + lane_off + (uint32_t)b * 64u + 32u, sv + 32);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(B_SFREE + b));
            const float w = rw[b * kRows + r];
            const int nvis = rn[b * kRows + r];
            const bool wide = tm[b].w != 0;
            uint32_t pk[32];
            if (w > 0.f) {
                chunk_softmax_row<kPolyPairEvery>(sv, nvis, w, sl2, pk, wide);
            } else {
#pragma unroll
                for (int x = 0; x < 32; ++x) pk[x] = 0u;
            }
            if (t >= 2 && !wait_warp(BAR(B_KVPFREE + b), ph ^ 1u, limit_ns, abort_flag, status)) break;
            unsigned char *prow = base + OFF_P + (size_t)b * kPTile + (size_t)r * 128;
#pragma unroll
            for (int pc = 0; pc < 8; ++pc)
                *reinterpret_cast<uint4 *>(prow + (((pc ^ (r & 7)) & 7) << 4)) =
                    make_uint4(pk[4 * pc], pk[4 * pc + 1], pk[4 * pc + 2], pk[4 * pc + 3]);
            fence_proxy_async_smem();
            mbar_arrive(BAR(B_PFULL + b));
        }
    } else if (warp >= 12) {
        // ---- epilogue: lane x of warp e holds column 32 e + x of every row's chunk output.  Half a tile
        // (64 rows) at a time: rows of d floats into the tile's query buffer, then one bulk reduction per
        // query (its G rows, contiguous in the buffer and in the accumulator)
        const int e = warp & 3;
        const uint32_t lane_off = (uint32_t)(32 * e) << 16;
        const int Gq = p.G;
        for (int t = 0; tile_of(t) < n_tiles; ++t) {
            const int b = t & 1;
            const uint32_t ph = (uint32_t)((t >> 1) & 1);
            bool ok = wait_warp(BAR(B_OFULL + b), ph, limit_ns, abort_flag, status) &&
                      wait_warp(BAR(B_ROW + b), ph, limit_ns, abort_flag, status);
            if (epilogue_bar_any(!ok || *abort_flag)) break;
            tc_fence_after();
            float *stage = reinterpret_cast<float *>(base + OFF_Q + (size_t)b * kQTile);   // [64][kD]
            const uint32_t stage_s = sQ + (uint32_t)b * kQTile;
            for (int half = 0; half < 2; ++half) {
#pragma unroll 1
                for (int cb = 0; cb < 2; ++cb) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_off + kColO + (uint32_t)b * 128u + 64u * (uint32_t)half + 32u * (uint32_t)cb, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) stage[(32 * cb + x) * kD + 32 * e + lane] = __uint_as_float(v[x]);
                }
                fence_proxy_async_smem();
                epilogue_bar_any(false);
                if (warp == 12 && lane == 0) {
                    const int q0 = 64 * half / Gq, q1 = 64 * (half + 1) / Gq;
                    for (int q = q0; q < q1; ++q) {
                        const int blk = rq[b * kRows + q];
                        if (blk >= 0)
                            bulk_reduce_add_f32(acc + (size_t)blk * Gq * kD, stage_s + (uint32_t)((q * Gq - 64 * half) * kD * 4),
                                                (uint32_t)(Gq * kD * 4));
                    }
                    asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group.read 0;" ::: "memory");
                }
                epilogue_bar_any(false);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(B_OFREE + b));
        }
        if (warp == 12 && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- the inversion ----------------------------------------------------------------------------------

struct CmPlan {
    int RQ, R;        // queries per range, ranges
    int M;            // lists: B * Hkv * R * nL
    int Mq;           // queries per tile
    long long max_tiles;
};

CmPlan cm_plan(const Dims &p)
{
    CmPlan c;
    c.Mq = kRows / p.G;
    // about 32 MB of float32 accumulator rows per range (G heads x d per query), a multiple of C queries
    long long rq = (32ll << 20) / ((long long)p.G * kD * 4);
    rq = rq / kC * kC;
    if (rq < kC) rq = kC;
    if (rq > p.N) rq = p.N;
    c.RQ = (int)rq;
    c.R = (p.N + c.RQ - 1) / c.RQ;
    c.M = p.B * p.Hkv * c.R * p.nL;
    const long long groups = (long long)p.B * p.Hkv * p.N;
    c.max_tiles = (groups * p.k + groups) / c.Mq + 2ll * c.M + 1;
    return c;
}

constexpr int kHistBins = 8192;   // shared-memory histogram of a block's lists (32 KB)

// The lists a block of consecutive query groups touches, (kv-group, range) pairs pr_lo .. pr_hi: when they
// fit the shared-memory histogram, the block counts there and adds each list's count to global memory
// once (the same few hundred lists are hit by every query of a block), else it counts in global memory.
__device__ __forceinline__ void block_pairs(const Dims &p, int RQ, int R, long long qg0, int &pr_lo, int &pr_hi)
{
    const long long groups = (long long)p.B * p.Hkv * p.N;
    const long long qa = qg0, qz = min(qg0 + (long long)blockDim.x, groups) - 1;
    pr_lo = (int)((qa / p.N) * R + (qa % p.N) / RQ);
    pr_hi = (int)((qz / p.N) * R + (qz % p.N) / RQ);
}

// per query group: count its selected chunks per (kv-group, range, chunk) list, and each head's
// log-sum-exp of its slot scores (the fusion weights' normaliser) and own chunk's fusion weight
__global__ void cm_count_kernel(Dims p, int RQ, int R, const int32_t *__restrict__ sel_idx,
                                const float *__restrict__ sel_score, int *__restrict__ cnt, float *__restrict__ lse,
                                float *__restrict__ ow)
{
    __shared__ int hist[kHistBins];
    const long long qg0 = (long long)blockIdx.x * blockDim.x, qg = qg0 + threadIdx.x;
    const bool valid = qg < (long long)p.B * p.Hkv * p.N;
    int pr_lo, pr_hi;
    block_pairs(p, RQ, R, qg0, pr_lo, pr_hi);
    const int span = (pr_hi - pr_lo + 1) * p.nL;
    const bool local = span <= kHistBins;
    if (local) {
        for (int x = threadIdx.x; x < span; x += blockDim.x) hist[x] = 0;
        __syncthreads();
    }
    if (valid) {
        const int i = (int)(qg % p.N);
        const long long bg = qg / p.N;
        const int b = (int)(bg / p.Hkv), g = (int)(bg % p.Hkv);
        const int pr = (int)(bg * R + i / RQ);
        for (int j = 0; j < p.k; ++j) {
            const int c = sel_idx[qg * p.k + j];
            if (c < 0) continue;
            if (local) atomicAdd(hist + (pr - pr_lo) * p.nL + c, 1);
            else atomicAdd(cnt + (size_t)pr * p.nL + c, 1);
        }
        const int ns = p.k + 1;
        for (int h = 0; h < p.G; ++h) {
            const size_t row = ((size_t)b * p.H + (size_t)g * p.G + h) * p.N + i;
            const float *sr = sel_score + row * ns;
            float m = -INFINITY;
            for (int j = 0; j < ns; ++j) m = fmaxf(m, sr[j]);
            float z = 0.f;
            for (int j = 0; j < ns; ++j) z += (sr[j] == -INFINITY) ? 0.f : __expf(sr[j] - m);
            const float l = m + __logf(z);
            lse[row] = l;
            ow[row] = __expf(sr[p.k] - l);   // the own chunk's fusion weight
        }
    }
    if (local) {
        __syncthreads();
        for (int x = threadIdx.x; x < span; x += blockDim.x)
            if (hist[x]) atomicAdd(cnt + (size_t)pr_lo * p.nL + x, hist[x]);
    }
}

// own-chunk queries of chunk c inside range r: [lo, hi)
__device__ __forceinline__ void own_range(const Dims &p, int RQ, int r, int c, int &lo, int &hi)
{
    const long long a = (long long)c * kC - p.q_offset, z = (long long)(c + 1) * kC - p.q_offset;
    lo = (int)max(max(a, (long long)r * RQ), 0ll);
    hi = (int)min(min(z, (long long)(r + 1) * RQ), (long long)p.N);
}

// Exclusive scans of the list sizes (entry offsets) and of the tiles per list, in three launches: each
// block of cm_scan_sums adds up its kScanSeg consecutive lists, cm_scan_top scans the block sums, and
// cm_scan_out scans each segment again from its block's offset.  Lists are read in rounds of 1024
// consecutive ones (coalesced), each round a block-wide scan.
constexpr int kScanSeg = 4096;   // lists per block: 4 rounds of 1024

__device__ __forceinline__ void list_size(const Dims &p, int RQ, int R, int Mq, int M, int m, const int *cnt,
                                          long long &ne, long long &nt)
{
    ne = 0;
    nt = 0;
    if (m >= M) return;
    const int c = m % p.nL, r = (m / p.nL) % R;
    int lo, hi;
    own_range(p, RQ, r, c, lo, hi);
    const int n_own = max(hi - lo, 0), n_ret = cnt[m];
    ne = n_ret;
    nt = (n_ret + Mq - 1) / Mq + (n_own + Mq - 1) / Mq;
}

// exclusive block-wide scan of two values per thread (1024 threads); the block totals in ta, tb
__device__ __forceinline__ void block_scan2(long long &a, long long &b, long long &ta, long long &tb)
{
    __shared__ long long wa[32], wb[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long xa = __shfl_up_sync(0xFFFFFFFFu, ia, o), xb = __shfl_up_sync(0xFFFFFFFFu, ib, o);
        if (lane >= o) {
            ia += xa;
            ib += xb;
        }
    }
    if (lane == 31) {
        wa[warp] = ia;
        wb[warp] = ib;
    }
    __syncthreads();
    if (warp == 0) {
        long long va = wa[lane], vb = wb[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long xa = __shfl_up_sync(0xFFFFFFFFu, va, o), xb = __shfl_up_sync(0xFFFFFFFFu, vb, o);
            if (lane >= o) {
                va += xa;
                vb += xb;
            }
        }
        wa[lane] = va;
        wb[lane] = vb;
    }
    __syncthreads();
    const long long pa = warp ? wa[warp - 1] : 0, pb = warp ? wb[warp - 1] : 0;
    ta = wa[31];
    tb = wb[31];
    a = pa + ia - a;
    b = pb + ib - b;
    __syncthreads();   // wa, wb are reused by the next call
}

__global__ void __launch_bounds__(1024) cm_scan_sums(Dims p, int RQ, int R, int Mq, int M, const int *__restrict__ cnt,
                                                     long long *__restrict__ bsum)
{
    long long se = 0, st = 0;
    for (int j = 0; j < kScanSeg / 1024; ++j) {
        long long ne, nt;
        list_size(p, RQ, R, Mq, M, blockIdx.x * kScanSeg + j * 1024 + threadIdx.x, cnt, ne, nt);
        long long te, tt;
        block_scan2(ne, nt, te, tt);
        se += te;
        st += tt;
    }
    if (threadIdx.x == 0) {
        bsum[2 * blockIdx.x] = se;
        bsum[2 * blockIdx.x + 1] = st;
    }
}

__global__ void __launch_bounds__(1024) cm_scan_top(int nb, long long *__restrict__ bsum, int *__restrict__ n_tiles)
{
    long long ce = 0, ct = 0;
    for (int base = 0; base < nb; base += 1024) {
        const int i = base + threadIdx.x;
        long long e = i < nb ? bsum[2 * i] : 0, t = i < nb ? bsum[2 * i + 1] : 0;
        long long te, tt;
        block_scan2(e, t, te, tt);
        if (i < nb) {
            bsum[2 * i] = ce + e;
            bsum[2 * i + 1] = ct + t;
        }
        ce += te;
        ct += tt;
    }
    if (threadIdx.x == 0) *n_tiles = (int)ct;
}

__global__ void __launch_bounds__(1024) cm_scan_out(Dims p, int RQ, int R, int Mq, int M, const int *__restrict__ cnt,
                                                    const long long *__restrict__ bsum, int *__restrict__ eoff,
                                                    int *__restrict__ fill, int *__restrict__ toff)
{
    long long ce = bsum[2 * blockIdx.x], ct = bsum[2 * blockIdx.x + 1];
    for (int j = 0; j < kScanSeg / 1024; ++j) {
        const int m = blockIdx.x * kScanSeg + j * 1024 + threadIdx.x;
        long long ne, nt;
        list_size(p, RQ, R, Mq, M, m, cnt, ne, nt);
        long long te, tt;
        block_scan2(ne, nt, te, tt);
        if (m < M) {
            eoff[m] = (int)(ce + ne);
            fill[m] = (int)(ce + ne);
            toff[m] = (int)(ct + nt);
        }
        ce += te;
        ct += tt;
    }
}

// tile descriptors of each list: its own-chunk tiles, then its retrieved tiles
__global__ void cm_tiles_kernel(Dims p, int RQ, int R, int Mq, int M, const int *__restrict__ cnt,
                                const int *__restrict__ eoff, const int *__restrict__ toff, int4 *__restrict__ tiles)
{
    const int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    const int c = m % p.nL, r = (m / p.nL) % R, bg = m / (p.nL * R);
    int lo, hi;
    own_range(p, RQ, r, c, lo, hi);
    const int n_own = max(hi - lo, 0), n_ret = cnt[m];
    int t = toff[m];
    for (int u = 0; u < n_own; u += Mq) tiles[t++] = make_int4(bg, c | kOwnBit, lo + u, min(Mq, n_own - u));
    for (int u = 0; u < n_ret; u += Mq) tiles[t++] = make_int4(bg, c, eoff[m] + u, min(Mq, n_ret - u));
}

// each selected (query, slot) into its chunk's list: entry = query << 6 | slot, and beside it the
// slot's fusion weight for each of the group's G heads.  Positions are reserved per list once per block
// (a shared-memory count, one global atomic per list, then shared-memory atomics), where the block's
// lists fit the histogram; otherwise one global atomic per entry.
__global__ void cm_scatter_kernel(Dims p, int RQ, int R, const int32_t *__restrict__ sel_idx,
                                  const float *__restrict__ sel_score, const float *__restrict__ lse,
                                  int *__restrict__ fill, int *__restrict__ entries, float *__restrict__ ew)
{
    __shared__ int hist[kHistBins];
    const long long qg0 = (long long)blockIdx.x * blockDim.x, qg = qg0 + threadIdx.x;
    const bool valid = qg < (long long)p.B * p.Hkv * p.N;
    int pr_lo, pr_hi;
    block_pairs(p, RQ, R, qg0, pr_lo, pr_hi);
    const int span = (pr_hi - pr_lo + 1) * p.nL;
    const bool local = span <= kHistBins;
    int i = 0, b = 0, g = 0, pr = 0;
    long long bg = 0;
    if (valid) {
        i = (int)(qg % p.N);
        bg = qg / p.N;
        b = (int)(bg / p.Hkv);
        g = (int)(bg % p.Hkv);
        pr = (int)(bg * R + i / RQ);
    }
    if (local) {
        for (int x = threadIdx.x; x < span; x += blockDim.x) hist[x] = 0;
        __syncthreads();
        if (valid)
            for (int j = 0; j < p.k; ++j) {
                const int c = sel_idx[qg * p.k + j];
                if (c >= 0) atomicAdd(hist + (pr - pr_lo) * p.nL + c, 1);
            }
        __syncthreads();
        for (int x = threadIdx.x; x < span; x += blockDim.x)
            if (hist[x]) hist[x] = atomicAdd(fill + (size_t)pr_lo * p.nL + x, hist[x]);
        __syncthreads();
    }
    if (!valid) return;
    const int ns = p.k + 1;
    for (int j = 0; j < p.k; ++j) {
        const int c = sel_idx[qg * p.k + j];
        if (c < 0) continue;
        const int at = local ? atomicAdd(hist + (pr - pr_lo) * p.nL + c, 1)
                             : atomicAdd(fill + (size_t)pr * p.nL + c, 1);
        entries[at] = (i << 6) | j;
        for (int h = 0; h < p.G; ++h) {
            const size_t row = ((size_t)b * p.H + (size_t)g * p.G + h) * p.N + i;
            ew[(size_t)at * p.G + h] = __expf(sel_score[row * ns + j] - lse[row]);
        }
    }
}

// the accumulator [B][Hkv][N][G][d] (float32) -> O [B][H][N][d], 8 elements per thread step
template <typename Tout>
__global__ void cm_finalize_kernel(Dims p, const float4 *__restrict__ acc, Tout *__restrict__ O)
{
    const size_t n8 = (size_t)p.B * p.H * p.N * kD / 8;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n8; e += (size_t)gridDim.x * blockDim.x) {
        const size_t o = e * 8, row = o / kD;           // O row (b H + h) N + i
        const int x = (int)(o % kD);
        const int i = (int)(row % p.N), bh = (int)(row / p.N), b = bh / p.H, h = bh % p.H;
        const int g = h / p.G, hh = h % p.G;
        const size_t src = ((((size_t)b * p.Hkv + g) * p.N + i) * p.G + hh) * kD + x;
        const float4 a = __ldg(acc + src / 4), z = __ldg(acc + src / 4 + 1);
        if constexpr (sizeof(Tout) == 4) {
            float4 *dst = reinterpret_cast<float4 *>(O + o);
            dst[0] = a;
            dst[1] = z;
        } else {
            __nv_bfloat162 v0 = __floats2bfloat162_rn(a.x, a.y), v1 = __floats2bfloat162_rn(a.z, a.w),
                           v2 = __floats2bfloat162_rn(z.x, z.y), v3 = __floats2bfloat162_rn(z.z, z.w);
            *reinterpret_cast<uint4 *>(O + o) =
                make_uint4(*reinterpret_cast<uint32_t *>(&v0), *reinterpret_cast<uint32_t *>(&v1),
                           *reinterpret_cast<uint32_t *>(&v2), *reinterpret_cast<uint32_t *>(&v3));
        }
    }
}

struct CmWs {
    int *cnt, *eoff, *fill, *toff, *n_tiles, *entries;
    long long *bsum;
    float *lse, *ow, *ew, *acc;
    int4 *tiles;
    size_t total;
};

CmWs cm_ws(const Dims &p, hils_dtype out, void *ws)
{
    const CmPlan c = cm_plan(p);
    CmWs w{};
    char *base = static_cast<char *>(ws);
    size_t off = attend_tc_ws_bytes(p);
    auto take = [&](size_t bytes) {
        char *ptr = base + off;
        off += align_up(bytes, 256);
        return ptr;
    };
    w.cnt = reinterpret_cast<int *>(take((size_t)c.M * 4));
    w.eoff = reinterpret_cast<int *>(take((size_t)c.M * 4));
    w.fill = reinterpret_cast<int *>(take((size_t)c.M * 4));
    w.toff = reinterpret_cast<int *>(take((size_t)c.M * 4));
    w.n_tiles = reinterpret_cast<int *>(take(4));
    w.bsum = reinterpret_cast<long long *>(take((size_t)((c.M + kScanSeg - 1) / kScanSeg) * 16));
    w.lse = reinterpret_cast<float *>(take((size_t)p.B * p.H * p.N * 4));
    w.ow = reinterpret_cast<float *>(take((size_t)p.B * p.H * p.N * 4));
    w.entries = reinterpret_cast<int *>(take((size_t)p.B * p.Hkv * p.N * p.k * 4 + 4));
    w.ew = reinterpret_cast<float *>(take((size_t)p.B * p.H * p.N * p.k * 4 + 4));
    w.tiles = reinterpret_cast<int4 *>(take((size_t)c.max_tiles * 16));
    w.acc = reinterpret_cast<float *>(take((size_t)p.B * p.H * p.N * kD * 4));
    w.total = off;
    return w;
}

}  // namespace

bool attend_cm_supported(const Dims &p, hils_dtype in)
{
    if (in != HILS_BF16 || p.d != kD || p.C != kC || p.N < 2 || p.k > 64) return false;
    if (p.G != 1 && p.G != 2 && p.G != 4 && p.G != 8 && p.G != 16) return false;
    if ((long long)p.N >= (1ll << 25)) return false;                                  // entry = query << 6 | slot
    if ((long long)p.B * p.H * p.N >= (1ll << 31)) return false;                      // accumulator rows as int
    return true;
}

// Chunk-major work grows with the selected pairs, the union kernel's with the chunks its query blocks
// cover; with uncorrelated selections a block covers about every visible chunk, so the union kernel
// does about (mean visible chunks) / (k + 1) times the useful work.  The chunk-major kernel pays a
// float32 reduction per selected pair and an inversion instead.  Measured on B200: at a ratio of
// about 4 (8K prefill, k = 16) the union kernel is 2.8 times faster, at about 62 (256K prefill,
// k = 32) the chunk-major kernel is 1.45 times faster; the switch is placed at 16, between the two.
bool attend_cm_preferred(const Dims &p)
{
    const double mean_visible = ((double)p.q_offset + 0.5 * p.N) / p.C + 0.5;
    return mean_visible > 16.0 * (p.k + 1);
}

size_t attend_cm_ws_bytes(const Dims &p, hils_dtype out) { return cm_ws(p, out, nullptr).total; }

cudaError_t launch_attend_prefill_cm(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                     const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                     const DeviceCtl &ctl, cudaStream_t s)
{
    const CmPlan c = cm_plan(p);
    const CmWs w = cm_ws(p, out, ws);
    cudaError_t e = launch_v_to_f16(p, V, ws, s);
    if (e != cudaSuccess) return e;
    const unsigned int *wide = reinterpret_cast<const unsigned int *>(
        static_cast<char *>(ws) + align_up((size_t)p.B * p.Hkv * p.T * kD * 2, 256));
    float *acc = w.acc;
    const long long groups = (long long)p.B * p.Hkv * p.N;
    e = cudaMemsetAsync(w.cnt, 0, (size_t)c.M * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(acc, 0, (size_t)p.B * p.H * p.N * kD * 4, s);
    if (e != cudaSuccess) return e;
    cm_count_kernel<<<(unsigned)((groups + 255) / 256), 256, 0, s>>>(p, c.RQ, c.R, sel_idx, sel_score, w.cnt, w.lse,
                                                                     w.ow);
    const int nb = (c.M + kScanSeg - 1) / kScanSeg;
    cm_scan_sums<<<nb, 1024, 0, s>>>(p, c.RQ, c.R, c.Mq, c.M, w.cnt, w.bsum);
    cm_scan_top<<<1, 1024, 0, s>>>(nb, w.bsum, w.n_tiles);
    cm_scan_out<<<nb, 1024, 0, s>>>(p, c.RQ, c.R, c.Mq, c.M, w.cnt, w.bsum, w.eoff, w.fill, w.toff);
    cm_tiles_kernel<<<(c.M + 255) / 256, 256, 0, s>>>(p, c.RQ, c.R, c.Mq, c.M, w.cnt, w.eoff, w.toff, w.tiles);
    cm_scatter_kernel<<<(unsigned)((groups + 255) / 256), 256, 0, s>>>(p, c.RQ, c.R, sel_idx, sel_score, w.lse,
                                                                       w.fill, w.entries, w.ew);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap tk, tv16, tvb;
    const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)p.B * p.Hkv * p.T};
    const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kC};
    if (!encode_tensor_map_sw128(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, 2, dims, strides, box) ||
        !encode_tensor_map_sw128(&tv16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws, 2, dims, strides, box) ||
        !encode_tensor_map_sw128(&tvb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, 2, dims, strides, box))
        return cudaErrorInvalidValue;
    static int n_sm = 0;
    if (!n_sm) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n_sm = 148;
    }
    e = cudaFuncSetAttribute(attend_cm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = (int)min((long long)n_sm, c.max_tiles);
    attend_cm_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(tk, tv16, tvb, p, static_cast<const __nv_bfloat16 *>(Q), w.ew,
                                                        w.ow, w.entries, w.tiles, w.n_tiles, wide, acc, ctl.status,
                                                        (unsigned long long)ctl.wait_limit);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (out == HILS_F32)
        cm_finalize_kernel<float><<<148 * 8, 256, 0, s>>>(p, reinterpret_cast<const float4 *>(acc), static_cast<float *>(O));
    else
        cm_finalize_kernel<__nv_bfloat16>
            <<<148 * 8, 256, 0, s>>>(p, reinterpret_cast<const float4 *>(acc), static_cast<__nv_bfloat16 *>(O));
    return cudaGetLastError();
}

}  // namespace hils
