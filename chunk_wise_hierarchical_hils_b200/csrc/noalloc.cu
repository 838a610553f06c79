// noalloc.cu -- decode selection with library-owned scratch, for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: plugins inside a host application that
// owns the whole device memory budget and exposes no allocator to them,
// processes whose memory is capped so that no per-call workspace can be
// reserved, and latency-critical paths that must never enter the driver's
// allocator (cudaMalloc may synchronise the device).  For them this entry
// point runs the same single-token decode selection kernel as
// hils_score_select, but takes the kernel's scratch (the per-split candidate
// lists and the completion tickets) from a fixed array that lives in the
// library's own device memory instead of a caller workspace.
//
// The array below is a __device__ variable.  Host code that names
// g_noalloc_scratch sees only the runtime's host-side shadow of it, not a device
// address, so the name is never passed to a kernel: the device address comes
// from cudaGetSymbolAddress, looked up once per device, with that device
// current, on the first call made on the device, and cached.  A device reset
// (cudaDeviceReset) ends the context that address belongs to; calls after one
// are not supported.  Every GPU that loads the library holds the array until the
// process exits.
#include <math.h>
#include <mutex>

#include "internal.h"

namespace hils {
namespace {

constexpr size_t kScratchBytes = HILS_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once).
hils_status scratch_on_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return HILS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return HILS_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return HILS_OK;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace
}  // namespace hils

using namespace hils;

extern "C" hils_status hils_decode_score_select_noalloc(const hils_problem *p, const void *Q, const void *L,
                                                        int32_t *sel_idx, float *sel_score, void *stream)
{
    Dims d;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    if (p->N != 1) return HILS_ERR_UNSUPPORTED;   // only the single-token decode kernel needs scratch
    if (!Q || !L || !sel_score || (p->k > 0 && !sel_idx)) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(L) || (sel_idx && !aligned16(sel_idx)) || !aligned16(sel_score))
        return HILS_ERR_INVALID_ARG;
    size_t need = 0;
    st = hils_score_select_workspace_size(p, &need);
    if (st != HILS_OK) return st;
    if (need > kScratchBytes) return HILS_ERR_WORKSPACE;   // problem too large for the fixed scratch
    void *scratch = nullptr;
    st = scratch_on_current_device(&scratch);
    if (st != HILS_OK) return st;
    DeviceCtl ctl;
    st = device_ctl(&ctl);
    if (st != HILS_OK) return st;
    // the launcher clears the completion tickets in the scratch before the kernel runs
    cudaError_t e = launch_select_decode(d, p->in_dtype, Q, L, sel_idx, sel_score, scratch, ctl,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}
