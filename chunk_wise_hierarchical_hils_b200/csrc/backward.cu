// backward.cu -- gradients of the HiLS forward pass through a fixed selection (CUDA cores, float32).
//
// "Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Sec. 3 Methodology, "Hierarchical
// softmax": the chunk retrieval scores enter the output as fusion weights, so the loss trains the
// landmarks and the retrieval through them, and a chunk that is not selected gets no gradient; the
// selection itself is a discrete choice, held fixed.  Per head h of kv-group g and query i at position
// p, over the slots c of its selection (retrieved chunks, then the own chunk):
//   forward   s_c = scale <q, L_c>,  w = softmax_c(s);  l_j = scale <q, k_j> (j in c, j <= p),
//             P^c = softmax_j(l) inside c,  o_c = sum_j P^c_j v_j,  o = sum_c w_c o_c;
//   backward  dw_c = <dO, o_c> = sum_j P^c_j u_j with u_j = <dO, v_j>;  ds_c = w_c (dw_c - sum w dw);
//             dq += scale sum_c ds_c L_c,  dL_c += scale ds_c q;
//             dP_j = w_c u_j and sum_j P^c_j dP_j = w_c dw_c, so dl_j = w_c P^c_j (u_j - dw_c);
//             dq += scale sum_j dl_j k_j,  dk_j += scale dl_j q,  dv_j += w_c P^c_j dO.
//
// One block per query group (b, g, i): the group's G heads share its selection.  Pass 1 stages each
// selected chunk's keys and values in shared memory and computes, per head, the chunk's softmax and
// dw_c; then the fusion weights and ds give the landmark terms; pass 2 stages the chunks again and
// adds the key and value terms.  dQ rows belong to their block and are written once; dK, dV and dL
// rows are shared by every query that selected their chunk and are accumulated with float32
// atomics (the call zeroes them first), so their summation order is not fixed.
#include <math.h>

#include "common.cuh"
#include "next_rows.h"

namespace hils {
namespace {

constexpr int NT = 256;

struct BwdLayout {
    size_t q, go, dq, ks, vs, pm, um, s, dw, w, ds, total;   // offsets in floats
};

__host__ __device__ inline BwdLayout bwd_layout(int G, int D, int C, int ns)
{
    BwdLayout L;
    L.q = 0;
    L.go = L.q + (size_t)G * D;
    L.dq = L.go + (size_t)G * D;
    L.ks = L.dq + (size_t)G * D;
    L.vs = L.ks + (size_t)C * D;
    L.pm = L.vs + (size_t)C * D;
    L.um = L.pm + (size_t)G * C;
    L.s = L.um + (size_t)G * C;
    L.dw = L.s + (size_t)G * ns;
    L.w = L.dw + (size_t)G * ns;
    L.ds = L.w + (size_t)G * ns;
    L.total = L.ds + (size_t)G * ns;
    return L;
}

// rows [0, n) of a D-wide row-major block, widened to float, into shared memory
template <typename Tin, int D>
__device__ __forceinline__ void stage_f32(float *dst, const Tin *src, int n)
{
    for (int e = threadIdx.x; e < n * (D / 8); e += NT) {
        float v[8];
        load8(src + (size_t)e * 8, v);
        float4 *o = reinterpret_cast<float4 *>(dst + (size_t)e * 8);
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// <a, b> over D elements of two shared-memory rows, the element order rotated by `rot` so that
// threads reading different rows at once hit different banks
template <int D>
__device__ __forceinline__ float dot_rot(const float *a, const float *b, int rot)
{
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int x = 0; x < D; x += 2) {
        const int x0 = (x + rot) & (D - 1), x1 = (x + 1 + rot) & (D - 1);
        s0 = fmaf(a[x0], b[x0], s0);
        s1 = fmaf(a[x1], b[x1], s1);
    }
    return s0 + s1;
}

template <typename Tin, int D>
__global__ void __launch_bounds__(NT) backward_kernel(Dims p, const Tin *__restrict__ Q, const Tin *__restrict__ K,
                                                      const Tin *__restrict__ V, const Tin *__restrict__ Lm,
                                                      const int32_t *__restrict__ sel_idx, const Tin *__restrict__ dO,
                                                      float *__restrict__ dQ, float *__restrict__ dK,
                                                      float *__restrict__ dV, float *__restrict__ dL)
{
    extern __shared__ __align__(16) float smf[];
    __shared__ int s_chunk[HILS_MAX_K + 1];
    const int G = p.G, C = p.C, ns = p.k + 1;
    const BwdLayout Ly = bwd_layout(G, D, C, ns);
    float *qs = smf + Ly.q, *gos = smf + Ly.go, *dqs = smf + Ly.dq, *Ks = smf + Ly.ks, *Vs = smf + Ly.vs;
    float *Pm = smf + Ly.pm, *Um = smf + Ly.um, *S = smf + Ly.s, *DW = smf + Ly.dw, *W = smf + Ly.w, *DS = smf + Ly.ds;

    const long long qg = blockIdx.x;
    const int i = (int)(qg % p.N), g = (int)((qg / p.N) % p.Hkv), b = (int)(qg / ((long long)p.N * p.Hkv));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long pos = (long long)p.q_offset + i;
    const int ci = (int)(pos / C);
    const size_t bg = (size_t)b * p.Hkv + g;

    for (int j = tid; j < ns; j += NT)
        s_chunk[j] = (j < p.k) ? sel_idx[(bg * p.N + i) * p.k + j] : ci;
    for (int e = tid; e < G * (D / 8); e += NT) {
        const int h = e / (D / 8), seg = e % (D / 8);
        const size_t row = (((size_t)b * p.H + (size_t)g * G + h) * p.N + i) * D;
        float v[8];
        load8(Q + row + seg * 8, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) qs[h * D + seg * 8 + u] = v[u];
        load8(dO + row + seg * 8, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) gos[h * D + seg * 8 + u] = v[u];
    }
    for (int e = tid; e < G * D; e += NT) dqs[e] = 0.f;
    __syncthreads();

    const Tin *Kbg = K + bg * (size_t)p.T * D, *Vbg = V + bg * (size_t)p.T * D, *Lbg = Lm + bg * (size_t)p.nL * D;

    // logits l (into Pm) and u = <dO, v_j> (into Um) of slot chunk c, n rows staged; then per head the
    // chunk softmax P (into Pm)
    auto chunk_softmax = [&](int n) {
        for (int t = tid; t < G * n; t += NT) {
            const int h = t / n, j = t % n;
            Pm[h * C + j] = p.scale * dot_rot<D>(qs + h * D, Ks + (size_t)j * D, j);
            Um[h * C + j] = dot_rot<D>(gos + h * D, Vs + (size_t)j * D, j);
        }
        __syncthreads();
        for (int h = warp; h < G; h += NT / 32) {
            float m = -INFINITY;
            for (int j = lane; j < n; j += 32) m = fmaxf(m, Pm[h * C + j]);
            m = warp_max(m);
            float z = 0.f;
            for (int j = lane; j < n; j += 32) {
                const float e = expf(Pm[h * C + j] - m);
                Pm[h * C + j] = e;
                z += e;
            }
            z = warp_sum(z);
            const float iz = 1.0f / z;
            for (int j = lane; j < n; j += 32) Pm[h * C + j] *= iz;
        }
        __syncthreads();
    };

    // ---- pass 1: dw_c and s_c of every slot ---------------------------------
    for (int jj = 0; jj < ns; ++jj) {
        const int c = s_chunk[jj];
        if (c < 0) {
            for (int h = tid; h < G; h += NT) {
                S[h * ns + jj] = -INFINITY;
                DW[h * ns + jj] = 0.f;
            }
            continue;
        }
        const int n = (int)min((long long)C, pos - (long long)c * C + 1);
        stage_f32<Tin, D>(Ks, Kbg + (size_t)c * C * D, n);
        stage_f32<Tin, D>(Vs, Vbg + (size_t)c * C * D, n);
        __syncthreads();
        chunk_softmax(n);
        for (int h = warp; h < G; h += NT / 32) {
            float a = 0.f;
            for (int j = lane; j < n; j += 32) a = fmaf(Pm[h * C + j], Um[h * C + j], a);
            a = warp_sum(a);
            float sc = 0.f;
            for (int x = lane; x < D; x += 32) sc = fmaf(qs[h * D + x], to_float(Lbg[(size_t)c * D + x]), sc);
            sc = warp_sum(sc);
            if (lane == 0) {
                DW[h * ns + jj] = a;
                S[h * ns + jj] = p.scale * sc;
            }
        }
        __syncthreads();
    }

    // ---- fusion weights, ds, and the landmark terms ----------------------------
    for (int h = warp; h < G; h += NT / 32) {
        float m = -INFINITY;
        for (int jj = lane; jj < ns; jj += 32) m = fmaxf(m, S[h * ns + jj]);
        m = warp_max(m);
        float z = 0.f;
        for (int jj = lane; jj < ns; jj += 32) z += (S[h * ns + jj] == -INFINITY) ? 0.f : expf(S[h * ns + jj] - m);
        z = warp_sum(z);
        float wdw = 0.f;
        for (int jj = lane; jj < ns; jj += 32) {
            const float wv = (S[h * ns + jj] == -INFINITY) ? 0.f : expf(S[h * ns + jj] - m) / z;
            W[h * ns + jj] = wv;
            wdw = fmaf(wv, DW[h * ns + jj], wdw);
        }
        wdw = warp_sum(wdw);
        for (int jj = lane; jj < ns; jj += 32) DS[h * ns + jj] = W[h * ns + jj] * (DW[h * ns + jj] - wdw);
    }
    __syncthreads();
    // dq += scale sum_c ds_c L_c (thread per (h, x)); dL_c += scale sum_h ds_c q_h (thread per (slot, x))
    for (int t = tid; t < G * D; t += NT) {
        const int h = t / D, x = t % D;
        float a = 0.f;
        for (int jj = 0; jj < ns; ++jj) {
            const int c = s_chunk[jj];
            if (c >= 0) a = fmaf(DS[h * ns + jj], to_float(Lbg[(size_t)c * D + x]), a);
        }
        dqs[t] += p.scale * a;
    }
    for (int t = tid; t < ns * D; t += NT) {
        const int jj = t / D, x = t % D;
        const int c = s_chunk[jj];
        if (c < 0) continue;
        float a = 0.f;
        for (int h = 0; h < G; ++h) a = fmaf(DS[h * ns + jj], qs[h * D + x], a);
        atomicAdd(dL + (bg * p.nL + c) * D + x, p.scale * a);
    }
    __syncthreads();

    // ---- pass 2: key and value terms --------------------------------------------
    for (int jj = 0; jj < ns; ++jj) {
        const int c = s_chunk[jj];
        if (c < 0) continue;
        const int n = (int)min((long long)C, pos - (long long)c * C + 1);
        stage_f32<Tin, D>(Ks, Kbg + (size_t)c * C * D, n);
        stage_f32<Tin, D>(Vs, Vbg + (size_t)c * C * D, n);
        __syncthreads();
        chunk_softmax(n);
        // Pm <- w_c P_j (the value weight), Um <- dl_j = w_c P_j (u_j - dw_c)
        for (int t = tid; t < G * n; t += NT) {
            const int h = t / n, j = t % n;
            const float wp = W[h * ns + jj] * Pm[h * C + j];
            Um[h * C + j] = wp * (Um[h * C + j] - DW[h * ns + jj]);
            Pm[h * C + j] = wp;
        }
        __syncthreads();
        for (int t = tid; t < G * D; t += NT) {
            const int h = t / D, x = t % D;
            float a = 0.f;
            for (int j = 0; j < n; ++j) a = fmaf(Um[h * C + j], Ks[(size_t)j * D + x], a);
            dqs[t] += p.scale * a;
        }
        for (int t = tid; t < n * D; t += NT) {
            const int j = t / D, x = t % D;
            float ak = 0.f, av = 0.f;
            for (int h = 0; h < G; ++h) {
                ak = fmaf(Um[h * C + j], qs[h * D + x], ak);
                av = fmaf(Pm[h * C + j], gos[h * D + x], av);
            }
            const size_t row = (bg * p.T + (size_t)c * C + j) * D + x;
            atomicAdd(dK + row, p.scale * ak);
            atomicAdd(dV + row, av);
        }
        __syncthreads();
    }

    for (int t = tid; t < G * D; t += NT) {
        const int h = t / D, x = t % D;
        dQ[(((size_t)b * p.H + (size_t)g * G + h) * p.N + i) * D + x] = dqs[t];
    }
}

template <typename Tin, int D>
cudaError_t launch_t(const Dims &p, const void *Q, const void *K, const void *V, const void *L,
                     const int32_t *sel_idx, const void *dO, float *dQ, float *dK, float *dV, float *dL,
                     cudaStream_t s)
{
    const size_t kv = (size_t)p.B * p.Hkv * p.T * D * sizeof(float);
    cudaError_t e = cudaMemsetAsync(dK, 0, kv, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dV, 0, kv, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dL, 0, (size_t)p.B * p.Hkv * p.nL * D * sizeof(float), s);
    if (e != cudaSuccess) return e;
    const size_t smem = bwd_layout(p.G, D, p.C, p.k + 1).total * sizeof(float);
    auto kern = backward_kernel<Tin, D>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long n_groups = (long long)p.B * p.Hkv * p.N;
    kern<<<(unsigned)n_groups, NT, smem, s>>>(p, static_cast<const Tin *>(Q), static_cast<const Tin *>(K),
                                              static_cast<const Tin *>(V), static_cast<const Tin *>(L), sel_idx,
                                              static_cast<const Tin *>(dO), dQ, dK, dV, dL);
    return cudaGetLastError();
}

}  // namespace

size_t backward_smem_bytes(const Dims &p) { return bwd_layout(p.G, p.d, p.C, p.k + 1).total * sizeof(float); }

cudaError_t launch_backward(const Dims &p, hils_dtype in, const void *Q, const void *K, const void *V, const void *L,
                            const int32_t *sel_idx, const void *dO, float *dQ, float *dK, float *dV, float *dL,
                            cudaStream_t s)
{
    if (in == HILS_F32)
        return p.d == 64 ? launch_t<float, 64>(p, Q, K, V, L, sel_idx, dO, dQ, dK, dV, dL, s)
                         : launch_t<float, 128>(p, Q, K, V, L, sel_idx, dO, dQ, dK, dV, dL, s);
    return p.d == 64 ? launch_t<__nv_bfloat16, 64>(p, Q, K, V, L, sel_idx, dO, dQ, dK, dV, dL, s)
                     : launch_t<__nv_bfloat16, 128>(p, Q, K, V, L, sel_idx, dO, dQ, dK, dV, dL, s);
}

}  // namespace hils
