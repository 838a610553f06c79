// decode_tiles.cuh -- one warp attends the query heads of a kv-group to one staged chunk on the tensor
// cores (mma.sync m16n8k16 tiles), for single-token decode.
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Abstract and Sec. 3 "Hierarchical
// softmax": softmax inside the chunk over the keys the query may see, the chunk output weighted by
// its fusion weight; Sec. 4 "Architecture": the group's heads share the chunk.
//
// The 16 rows of the tiles are the group's G query heads (zero padded): S = Q K_c^T in float32, the
// row softmax scaled by the row's fusion weight, then O += P V_c with P split into a bf16 high part
// and a bf16 remainder (so P keeps about 16 bits).  K and V are C x 128 bf16 tiles written by TMA with
// the 128-byte swizzle as two 64-column halves, read with ldmatrix (V transposed).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace hils {
namespace dtiles {

constexpr int kQPitch = 272;   // bytes per staged Q row (256 + 16: ldmatrix rows on distinct banks)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D (16x8 f32) += A (16x16 bf16, row-major fragment) * B (16x8 bf16, column-major fragment)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// A tile written by TMA with the 128-byte swizzle: rows of 128 bytes, the 16-byte piece j of row r
// stored at piece j ^ (r % 8).
__device__ __forceinline__ uint32_t sw128(uint32_t tile, int r, int j)
{
    return tile + (uint32_t)r * 128u + ((uint32_t)(j ^ (r & 7)) << 4);
}

// One warp: oacc (rows gid and gid + 8 of the 16, columns nd * 8 + 2 tig + {0, 1}) += w * softmax(S) V
// over chunk tiles kt (keys) and vt (values), each two 64-column halves of C rows (C * 128 bytes);
// qs = the 16 staged query rows (kQPitch apart); n_vis = keys the query may see; sl2 = scale * log2 e;
// w0 / w1 = fusion weights of rows gid / gid + 8 (0 for padding rows).
template <int C>
__device__ __forceinline__ void warp_chunk_mma(uint32_t qs, uint32_t kt, uint32_t vt, int n_vis, float sl2, float w0,
                                               float w1, float (&oacc)[16][4])
{
    constexpr uint32_t HALF = C * 128;
    constexpr int NT = C / 8;   // key tiles of 8
    const int lane = threadIdx.x & 31, tig = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;   // ldmatrix: the matrix and row this lane addresses

    // S = Q K^T: 16 rows x C keys
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
    for (int ks2 = 0; ks2 < 4; ++ks2) {
        // Q fragments of k-steps 2 ks2 and 2 ks2 + 1 (d = 32 ks2 .. 32 ks2 + 31)
        uint32_t qa[2][4];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int ks = 2 * ks2 + h2;
            const uint32_t qaddr = qs + (uint32_t)((rr + 8 * (mi & 1)) * kQPitch + (ks * 16 + 8 * (mi >> 1)) * 2);
            ldsm_x4(qaddr, qa[h2][0], qa[h2][1], qa[h2][2], qa[h2][3]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int key = nt * 8 + rr, dc = 4 * ks2 + mi;   // 16-byte piece of d
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sw128(kt + (uint32_t)(dc >> 3) * HALF, key, dc & 7), b0, b1, b2, b3);
            mma16816(sacc[nt], qa[0], b0, b1);
            mma16816(sacc[nt], qa[1], b2, b3);
        }
    }

    // softmax per row (rows gid and gid + 8), scaled by the row's fusion weight
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int key = nt * 8 + tig * 2 + e;
            if (key >= n_vis) {
                sacc[nt][e] = -INFINITY;
                sacc[nt][2 + e] = -INFINITY;
            }
            m0 = fmaxf(m0, sacc[nt][e]);
            m1 = fmaxf(m1, sacc[nt][2 + e]);
        }
    m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, 1));
    m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, 2));
    m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, 1));
    m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, 2));
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            sacc[nt][e] = exp2f((sacc[nt][e] - m0) * sl2);
            sacc[nt][2 + e] = exp2f((sacc[nt][2 + e] - m1) * sl2);
            l0 += sacc[nt][e];
            l1 += sacc[nt][2 + e];
        }
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    const float f0 = w0 / l0, f1 = w1 / l1;

    // O += P V over the chunk's keys, 16 per k-step; P = high + remainder, both bf16
#pragma unroll
    for (int kk = 0; kk < C / 16; ++kk) {
        float pv[8];
        pv[0] = sacc[2 * kk][0] * f0;
        pv[1] = sacc[2 * kk][1] * f0;
        pv[2] = sacc[2 * kk][2] * f1;
        pv[3] = sacc[2 * kk][3] * f1;
        pv[4] = sacc[2 * kk + 1][0] * f0;
        pv[5] = sacc[2 * kk + 1][1] * f0;
        pv[6] = sacc[2 * kk + 1][2] * f1;
        pv[7] = sacc[2 * kk + 1][3] * f1;
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            ph[q] = pack_bf16(pv[2 * q], pv[2 * q + 1]);
            const __nv_bfloat162 hv = *reinterpret_cast<const __nv_bfloat162 *>(&ph[q]);
            pl[q] = pack_bf16(pv[2 * q] - __low2float(hv), pv[2 * q + 1] - __high2float(hv));
        }
#pragma unroll
        for (int nd2 = 0; nd2 < 8; ++nd2) {
            const int key = kk * 16 + rr + 8 * (mi & 1), dc = 2 * nd2 + (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sw128(vt + (uint32_t)(dc >> 3) * HALF, key, dc & 7), b0, b1, b2, b3);
            mma16816(oacc[2 * nd2], ph, b0, b1);
            mma16816(oacc[2 * nd2], pl, b0, b1);
            mma16816(oacc[2 * nd2 + 1], ph, b2, b3);
            mma16816(oacc[2 * nd2 + 1], pl, b2, b3);
        }
    }
}

}  // namespace dtiles
}  // namespace hils
