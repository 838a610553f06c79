// gen_cuda.cu -- CUDA twin of synth/philox.py and synth/workloads.py.
//
// Fills whole input tensors on the device with exactly the values the numpy
// recipe produces (Philox4x32-10, Box-Muller, the same float64 operation
// order with fused multiply-add excluded, then float32 and bfloat16 rounding,
// both nearest-even).  Test and benchmark infrastructure only; it has no part
// of the attention computation.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

extern "C" {
typedef struct {
    int B, H, Hkv, N, T, d, C, q_offset;
    int dtype;                 // 0 float32, 1 bfloat16
    unsigned long long seed;
    int input_scale;           // multiply deviates by 1/sqrt(sqrt(d))
    int l_mode;                // 0 i.i.d., 1 chunk mean of keys + noise
    double l_noise;
    int n_needles, needle_period;
    double needle_shift;
} synth_params;
}

namespace {

enum { S_Q = 1, S_K = 2, S_V = 3, S_L = 4, S_LNOISE = 5, S_U = 6, S_NEEDLE = 7 };

__device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    }
}

__device__ __forceinline__ void block_words(unsigned long long seed, uint32_t stream, uint64_t n, uint32_t *x0,
                                            uint32_t *x1)
{
    uint32_t c[4] = {(uint32_t)n, (uint32_t)(n >> 32), 0u, 0u};
    philox4x32_10(c, (uint32_t)seed, stream);
    *x0 = c[0];
    *x1 = c[1];
}

__device__ __forceinline__ double gaussian(unsigned long long seed, uint32_t stream, uint64_t e)
{
    uint32_t x0, x1;
    block_words(seed, stream, e >> 1, &x0, &x1);
    const double inv = 2.3283064365386963e-10;
    const double u1 = __dmul_rn(__dadd_rn((double)x0, 0.5), inv);
    const double u2 = __dmul_rn(__dadd_rn((double)x1, 0.5), inv);
    const double r = sqrt(__dmul_rn(-2.0, log(u1)));
    const double th = __dmul_rn(6.283185307179586, u2);
    return (e & 1) ? __dmul_rn(r, sin(th)) : __dmul_rn(r, cos(th));
}

__device__ __forceinline__ double uniform(unsigned long long seed, uint32_t stream, uint64_t idx)
{
    uint32_t x0, x1;
    block_words(seed, stream, idx, &x0, &x1);
    return __dmul_rn(__dadd_rn((double)x0, 0.5), 2.3283064365386963e-10);
}

__device__ __forceinline__ void store(const synth_params &p, void *out, size_t e, double v)
{
    const float f = __double2float_rn(v);
    if (p.dtype == 0) static_cast<float *>(out)[e] = f;
    else static_cast<__nv_bfloat16 *>(out)[e] = __float2bfloat16_rn(f);
}

__device__ __forceinline__ double widen(const synth_params &p, const void *buf, size_t e)
{
    if (p.dtype == 0) return (double)static_cast<const float *>(buf)[e];
    return (double)__bfloat162float(static_cast<const __nv_bfloat16 *>(buf)[e]);
}

// u[g][j] unit vectors (sequential sum of squares) and needle chunk lists
__global__ void setup_kernel(synth_params p, double *u, int *needles)
{
    const int g = blockIdx.x;
    if (threadIdx.x == 0) {
        double ss = 0.0;
        for (int j = 0; j < p.d; ++j) {
            const double z = gaussian(p.seed, S_U, (uint64_t)g * p.d + j);
            u[(size_t)g * p.d + j] = z;
            ss = __dadd_rn(ss, __dmul_rn(z, z));
        }
        const double nrm = sqrt(ss);
        for (int j = 0; j < p.d; ++j) u[(size_t)g * p.d + j] = u[(size_t)g * p.d + j] / nrm;
        if (p.n_needles) {
            const int width = (p.T / p.C) / p.n_needles;
            for (int m = 0; m < p.n_needles; ++m) {
                const double x = uniform(p.seed, S_NEEDLE, (uint64_t)g * p.n_needles + m);
                needles[g * p.n_needles + m] = m * width + (int)floor(__dmul_rn(x, (double)width));
            }
        }
    }
}

__device__ __forceinline__ double in_scale(const synth_params &p)
{
    return p.input_scale ? 1.0 / sqrt(sqrt((double)p.d)) : 1.0;
}

__device__ bool is_needle(const synth_params &p, const int *needles, int g, long long chunk)
{
    if (!p.n_needles) return false;
    // needle chunks are sorted (one per stratum): binary search
    int lo = 0, hi = p.n_needles - 1;
    const int *a = needles + g * p.n_needles;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] == chunk) return true;
        if (a[mid] < chunk) lo = mid + 1; else hi = mid - 1;
    }
    return false;
}

__global__ void fill_q_kernel(synth_params p, const double *u, void *out, size_t n)
{
    const double sc = in_scale(p);
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        double v = gaussian(p.seed, S_Q, e);
        if (p.input_scale) v = __dmul_rn(v, sc);
        if (p.n_needles) {
            const int x = (int)(e % p.d);
            const long long i = (long long)((e / p.d) % p.N);
            const int h = (int)((e / ((size_t)p.d * p.N)) % p.H);
            if (((long long)p.q_offset + i) % p.needle_period == 0) {
                const int g = h / (p.H / p.Hkv);
                v = __dadd_rn(v, __dmul_rn(p.needle_shift, u[(size_t)g * p.d + x]));
            }
        }
        store(p, out, e, v);
    }
}

__global__ void fill_kv_kernel(synth_params p, int stream, const double *u, const int *needles, void *out, size_t n)
{
    const double sc = in_scale(p);
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        double v = gaussian(p.seed, (uint32_t)stream, e);
        if (p.input_scale) v = __dmul_rn(v, sc);
        if (stream == S_K && p.n_needles) {
            const int x = (int)(e % p.d);
            const long long t = (long long)((e / p.d) % p.T);
            const int g = (int)((e / ((size_t)p.d * p.T)) % p.Hkv);
            if (is_needle(p, needles, g, t / p.C)) v = __dadd_rn(v, __dmul_rn(p.needle_shift, u[(size_t)g * p.d + x]));
        }
        store(p, out, e, v);
    }
}

__global__ void fill_l_kernel(synth_params p, const double *u, const int *needles, const void *K, void *out, size_t n)
{
    const int nL = (p.T + p.C - 1) / p.C;
    const double sc = in_scale(p);
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int x = (int)(e % p.d);
        const long long c = (long long)((e / p.d) % nL);
        const size_t bg = e / ((size_t)p.d * nL);
        const int g = (int)(bg % p.Hkv);
        double v;
        if (p.l_mode == 1) {
            const long long t0 = c * p.C;
            const int rows = (int)min((long long)p.C, (long long)p.T - t0);
            double acc = widen(p, K, (bg * p.T + t0) * p.d + x);
            for (int r = 1; r < rows; ++r) acc = __dadd_rn(acc, widen(p, K, (bg * p.T + t0 + r) * p.d + x));
            const double mean = acc / (double)rows;
            v = __dadd_rn(mean, __dmul_rn(p.l_noise, gaussian(p.seed, S_LNOISE, e)));
        } else {
            v = gaussian(p.seed, S_L, e);
            if (p.input_scale) v = __dmul_rn(v, sc);
            if (is_needle(p, needles, g, c)) v = __dadd_rn(v, __dmul_rn(p.needle_shift, u[(size_t)g * p.d + x]));
        }
        store(p, out, e, v);
    }
}

int grid_for(size_t n) { return (int)(n / 256 + 1 < 148 * 64 ? n / 256 + 1 : 148 * 64); }

}  // namespace

extern "C" {

// Fills Q [B,H,N,d], K and V [B,Hkv,T,d] and L [B,Hkv,ceil(T/C),d] (any may be
// NULL except that chunk-mean landmarks need K).  Synchronous; returns a
// cudaError_t value.
__attribute__((visibility("default"))) int synth_fill(const synth_params *pp, void *Q, void *K, void *V, void *L)
{
    const synth_params p = *pp;
    double *u = nullptr;
    int *needles = nullptr;
    cudaError_t e = cudaMalloc(&u, sizeof(double) * (size_t)p.Hkv * p.d);
    if (e != cudaSuccess) return (int)e;
    e = cudaMalloc(&needles, sizeof(int) * (size_t)p.Hkv * (p.n_needles > 0 ? p.n_needles : 1));
    if (e != cudaSuccess) { cudaFree(u); return (int)e; }
    setup_kernel<<<p.Hkv, 32>>>(p, u, needles);
    const size_t nq = (size_t)p.B * p.H * p.N * p.d;
    const size_t nkv = (size_t)p.B * p.Hkv * p.T * p.d;
    const size_t nl = (size_t)p.B * p.Hkv * ((p.T + p.C - 1) / p.C) * p.d;
    if (Q) fill_q_kernel<<<grid_for(nq), 256>>>(p, u, Q, nq);
    if (K) fill_kv_kernel<<<grid_for(nkv), 256>>>(p, S_K, u, needles, K, nkv);
    if (V) fill_kv_kernel<<<grid_for(nkv), 256>>>(p, S_V, u, needles, V, nkv);
    if (L) {
        if (p.l_mode == 1 && !K) { cudaFree(u); cudaFree(needles); return (int)cudaErrorInvalidValue; }
        fill_l_kernel<<<grid_for(nl), 256>>>(p, u, needles, K, L, nl);
    }
    e = cudaGetLastError();
    cudaError_t e2 = cudaDeviceSynchronize();
    cudaFree(u);
    cudaFree(needles);
    return (int)(e != cudaSuccess ? e : e2);
}

}  // extern "C"
