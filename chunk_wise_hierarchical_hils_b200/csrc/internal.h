// internal.h -- resolved problem description and kernel launchers (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/hils.h"

namespace hils {

// Problem with derived quantities, passed by value to every kernel.
struct Dims {
    int B, H, Hkv, G;
    int N, T, d, C, k;
    int nL;          // landmarks per sequence, ceil(T / C)
    int q_offset;
    float scale;     // resolved: never 0
};

// Checks a problem description and derives its quantities (the validation of every entry point).
hils_status resolve(const hils_problem *p, Dims *o);

// Device-side status shared by all kernels of the library.
struct DeviceCtl {
    unsigned int *status;   // HILS_OK or HILS_ERR_TIMEOUT, sticky until read
    long long wait_limit;   // ns a bounded wait may take before it gives up
    int inject_stall;       // test control: tensor-core kernels wait once on a barrier nothing signals
};

// Decode selection layout in the workspace.
struct DecodePlan {
    int spl;        // candidate chunks per split CTA (power of two)
    int nsplit;     // split CTAs per (b, g)
    int sort_n;     // power of two >= max(spl, nsplit * k)
    int slots_per_cta;  // attend: selected chunks per CTA
    int nsplit2;        // attend: CTAs per (b, g)
};

DecodePlan decode_plan(const Dims &p);
size_t decode_select_ws_bytes(const Dims &p);
size_t decode_attend_ws_bytes(const Dims &p);

// Launchers return the cudaGetLastError() of their launch.
cudaError_t launch_select_prefill(const Dims &p, hils_dtype in, const void *Q, const void *L,
                                  int32_t *sel_idx, float *sel_score, cudaStream_t s);
cudaError_t launch_select_decode(const Dims &p, hils_dtype in, const void *Q, const void *L,
                                 int32_t *sel_idx, float *sel_score, void *ws, const DeviceCtl &ctl,
                                 cudaStream_t s);
size_t decode_select_smem_bytes(const Dims &p, hils_dtype in);
cudaError_t launch_attend_prefill(const Dims &p, hils_dtype in, hils_dtype out, const void *Q,
                                  const void *K, const void *V, const int32_t *sel_idx,
                                  const float *sel_score, void *O, void *ws, const DeviceCtl &ctl,
                                  cudaStream_t s);
cudaError_t launch_attend_prefill_simt(const Dims &p, hils_dtype in, hils_dtype out, const void *Q,
                                       const void *K, const void *V, const int32_t *sel_idx,
                                       const float *sel_score, void *O, cudaStream_t s);
bool attend_tc_supported(const Dims &p, hils_dtype in);
bool select_tc_supported(const Dims &p, hils_dtype in);
bool select_tc_resident(const Dims &p);   // the heads kernel keeps every landmark tile in TMEM
cudaError_t launch_select_prefill_tc(const Dims &p, const void *Q, const void *L, int32_t *sel_idx,
                                     float *sel_score, const DeviceCtl &ctl, cudaStream_t s);
// Prefill selection with one product row per query (group score from the mean query): bf16, d = 128, k <= 32.
// With wc > 1 or a bias [B][Hkv][nL] it writes the windowed selection (k + wc - 1 past slots per row).
bool select_q_supported(const Dims &p, hils_dtype in, int wc = 1);
bool select_q_preferred(const Dims &p);   // where it beats the kernel with a row per head
cudaError_t launch_select_prefill_q(const Dims &p, const void *Q, const void *L, int32_t *sel_idx, float *sel_score,
                                    const DeviceCtl &ctl, cudaStream_t s, int wc = 1, const float *bias = nullptr);
size_t attend_tc_ws_bytes(const Dims &p);   // V as f16 + one flag word per (b, kv-head): launch_v_to_f16's output
// V (bf16) converted to f16 at the start of ws, and per (b, kv-head) a flag set when a value's magnitude
// is 65536 or more (the slice then takes a bf16 value product with V as given).
cudaError_t launch_v_to_f16(const Dims &p, const void *V, void *ws, cudaStream_t s);
const unsigned int *attend_tc_wide_flags(const Dims &p, const void *ws);   // launch_v_to_f16's flag words in ws
// The same attention as a persistent kernel (one CTA per SM walking query tiles); same workspace.
bool attend_tc_persistent_supported(const Dims &p, hils_dtype in);
cudaError_t launch_attend_prefill_tc_persistent(const Dims &p, hils_dtype out, const void *Q, const void *K,
                                                const void *V, const int32_t *sel_idx, const float *sel_score,
                                                void *O, void *ws, const DeviceCtl &ctl, cudaStream_t s);
// Chunk-major prefill attention (selection inverted per chunk, tiles of gathered query rows, partial
// outputs added in L2): bf16, d = 128, C = 64.
bool attend_cm_supported(const Dims &p, hils_dtype in);
bool attend_cm_preferred(const Dims &p);
size_t attend_cm_ws_bytes(const Dims &p, hils_dtype out);
cudaError_t launch_attend_prefill_cm(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                     const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                     const DeviceCtl &ctl, cudaStream_t s);
cudaError_t launch_attend_prefill_tc(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                     const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                     const DeviceCtl &ctl, cudaStream_t s);
cudaError_t launch_attend_decode(const Dims &p, hils_dtype in, hils_dtype out, const void *Q,
                                 const void *K, const void *V, const int32_t *sel_idx,
                                 const float *sel_score, void *O, void *ws, const DeviceCtl &ctl,
                                 cudaStream_t s);

// Single-token decode attention on the tensor cores (mma.sync tiles): bf16, d = 128, C in {64, 128}.
bool attend_decode_mma_supported(const Dims &p, hils_dtype in);
cudaError_t launch_attend_decode_mma(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                     const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                     const DeviceCtl &ctl, cudaStream_t s);

// Single-token decode in one cooperative kernel (selection and attention): bf16, d = 128, C = 64, with
// B * Hkv no more than the SM count.  Writes sel_idx / sel_score (N == 1 rows) as well as O.
bool decode_fused_supported(const Dims &p, hils_dtype in);
size_t decode_fused_ws_bytes(const Dims &p);
cudaError_t launch_decode_fused(const Dims &p, hils_dtype out, const void *Q, const void *K, const void *V,
                                const void *L, int32_t *sel_idx, float *sel_score, void *O, void *ws,
                                const DeviceCtl &ctl, cudaStream_t s);

// TMA tile map (no interleave, 128-byte swizzle, 256-byte L2 promotion, zero fill out of bounds); rank 1..3,
// strides in bytes for dimensions 1..rank-1.  False when the driver's encoder is missing or rejects the map.
bool encode_tensor_map_sw128(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, int rank,
                             const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box);

// Device status word and wait limit of the current device (looked up once per device).
hils_status device_ctl(DeviceCtl *ctl);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace hils
