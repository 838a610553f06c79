// next_rows.h -- launchers of the method's extensions beyond the forward path (not part of the ABI):
// the local window with a per-chunk bias, landmark generation, the backward pass, and the debug check
// of a caller's selection.  Kept apart from internal.h so that the forward path's kernels do not depend on them.
#pragma once

#include "internal.h"

namespace hils {

// Selection with a local window of wc chunks and an optional per-chunk bias (float [B][Hkv][nL]):
// sel_idx rows of k + wc - 1 past slots, sel_score rows of k + wc (see select_window.cu).
cudaError_t launch_select_window(const Dims &p, hils_dtype in, int wc, const float *bias, const void *Q,
                                 const void *L, int32_t *sel_idx, float *sel_score, cudaStream_t s);

// Debug check of a caller-supplied selection (entries -1 or past chunks of their query, no repeats in a
// row): runs a kernel on s, waits for it and returns HILS_ERR_INVALID_ARG when a row breaks the rule.
hils_status check_selection(const Dims &p, const int32_t *sel_idx, cudaStream_t s);

// Landmark generation for chunks [c_begin, c_end) of every (b, g): one warp per chunk, key rows read once.
bool landmarks_launchable(long long B, long long Hkv, int span);
cudaError_t launch_landmarks(int B, int Hkv, int T, int d, int C, float scale, hils_dtype in, const void *K,
                             const void *U, void *L, float *beta, int c_begin, int c_end, cudaStream_t s);

// Gradients through a fixed selection (float32 outputs; dK, dV and dL zeroed, then accumulated).
size_t backward_smem_bytes(const Dims &p);
cudaError_t launch_backward(const Dims &p, hils_dtype in, const void *Q, const void *K, const void *V, const void *L,
                            const int32_t *sel_idx, const void *dO, float *dQ, float *dK, float *dV, float *dL,
                            cudaStream_t s);

}  // namespace hils
