// check_selection.cu -- debug check of a caller-supplied selection before chunk attention.
//
// hils_chunk_attend_fuse takes sel_idx from its caller.  Every entry must be -1 or a past chunk of its
// query (0 <= c < c_i, c_i = floor((q_offset + i) / C)), and a row must not name a chunk twice: the
// attention gathers each listed chunk and fuses it once per slot.  The attention kernels trust this;
// with the check switched on the library first runs this kernel, reads its verdict and refuses the
// call (nothing else launched) when any row breaks the rule.
#include "common.cuh"
#include "next_rows.h"

namespace hils {
namespace {

// One thread per (b, g, i) row; a violation sets *bad.
__global__ void check_selection_kernel(Dims p, const int32_t *__restrict__ sel_idx, unsigned int *bad)
{
    const long long rows = (long long)p.B * p.Hkv * p.N;
    for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < rows;
         r += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(r % p.N);
        const int ci = (int)(((long long)p.q_offset + i) / p.C);
        const int32_t *row = sel_idx + r * p.k;
        bool ok = true;
        for (int j = 0; j < p.k && ok; ++j) {
            const int c = row[j];
            if (c == -1) continue;
            if (c < 0 || c >= ci) ok = false;
            for (int j2 = 0; j2 < j && ok; ++j2) ok = row[j2] != c;
        }
        if (!ok) atomicOr(bad, 1u);
    }
}

}  // namespace

namespace {

__device__ unsigned int g_sel_bad;   // the check's verdict (one word per device)

}  // namespace

hils_status check_selection(const Dims &p, const int32_t *sel_idx, cudaStream_t s)
{
    if (p.k == 0) return HILS_OK;
    unsigned int *bad = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&bad), g_sel_bad) != cudaSuccess) return HILS_ERR_CUDA;
    if (cudaMemsetAsync(bad, 0, sizeof(unsigned int), s) != cudaSuccess) return HILS_ERR_CUDA;
    const long long rows = (long long)p.B * p.Hkv * p.N;
    const long long blocks = (rows + 255) / 256;
    check_selection_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, s>>>(p, sel_idx, bad);
    if (cudaGetLastError() != cudaSuccess) return HILS_ERR_CUDA;
    unsigned int verdict = 0;
    if (cudaMemcpyAsync(&verdict, bad, sizeof(verdict), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return HILS_ERR_CUDA;
    return verdict ? HILS_ERR_INVALID_ARG : HILS_OK;
}

}  // namespace hils
