// tensor_map.cu -- host-side encoding of TMA tensor maps (tile mode, 128-byte swizzle).
//
// The driver's encoder is looked up through the runtime, so the library does not link against
// libcuda (it loads on machines without a GPU driver; the lookup happens on the first launch).
#include <cuda.h>

#include "internal.h"

namespace hils {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder()
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

bool encode_tensor_map_sw128(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, int rank,
                             const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box)
{
    EncodeTiledFn fn = encoder();
    if (!fn || rank < 1 || rank > 3) return false;
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, dt, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace hils
