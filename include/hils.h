/*
 * hils.h -- C ABI of the HiLS attention forward library (libhils.so), sm_100a.
 *
 * Hierarchical Landmark Sparse (HiLS) attention, as described in
 * "Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling"
 * (arXiv 2607.02980v1, summary page):
 *   - Abstract: each query attends independently inside every retrieved chunk;
 *     the per-chunk outputs are fused according to chunk retrieval scores.
 *   - Sec. 3 Methodology, "Sparse training": each query scores all chunk
 *     summaries (landmarks) and keeps the top-K chunks.
 *   - Sec. 3 Methodology, "Hierarchical softmax": softmax inside each chunk,
 *     then a softmax over the chunks' surrogate masses fuses the chunk outputs.
 *   - Sec. 4 Practical Design Choices, "Architecture": under GQA the heads of a
 *     group share one retrieved chunk set, gathered once.
 *   - Sec. 2 Preliminary: chunks are a uniform partition of the sequence.
 *
 * Definition computed (query i at position p = q_offset + i, own chunk
 * c_i = floor(p / C), head h in kv-group g = h / (H / Hkv), scale s):
 *   1. retrieval score  s_{h,c} = s * <q_{h,i}, L_{g,c}>;
 *      group score      S_{g,c} = mean over the group's heads of s_{h,c}.
 *   2. selection: the min(k, c_i) past chunks c < c_i with the largest group
 *      scores (equal scores: lower chunk index first), in rank order; the own
 *      chunk c_i is always added as slot k.
 *   3. inside each selected chunk: softmax over the tokens c*C .. c*C+C-1 that
 *      are at positions <= p, of s * <q, k_j>; chunk output o_c = sum p_j v_j.
 *   4. fusion weights w_{h,c} = softmax over the selected slots of s_{h,c};
 *      output o_{h,i} = sum_c w_{h,c} o_c.
 *
 * Tensor layouts (all row-major, contiguous, device memory, 16-byte aligned):
 *   Q  [B][H][N][d]        in_dtype
 *   K  [B][Hkv][T][d]      in_dtype
 *   V  [B][Hkv][T][d]      in_dtype
 *   L  [B][Hkv][nL][d]     in_dtype, nL = ceil(T / C), row c = landmark of chunk c
 *   O  [B][H][N][d]        out_dtype
 *   sel_idx   [B][Hkv][N][k]   int32: selected past chunks in rank order, -1 padded
 *   sel_score [B][H][N][k+1]   float: s_{h,c} of each slot (slot k = own chunk),
 *                              -INFINITY for empty slots
 * Prefill: q_offset = 0, N = T.  Single-token decode: N = 1, q_offset = T - 1
 * (the new token's key/value already at position T-1; the landmark of a partial
 * last chunk is supplied by the caller).  Any 0 <= q_offset, q_offset + N <= T
 * is accepted.
 *
 * Ownership: the caller allocates and owns every buffer, including the
 * workspace; the library allocates no device memory on these calls.
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream) and validate their arguments before any launch: a status other than
 * HILS_OK from the call itself means nothing was launched.  Device-side
 * failures of bounded waits are reported by hils_sync_status().
 * Thread safety: calls may come from several host threads; kernels that share
 * one workspace must not overlap on the GPU.
 * Device state: the library looks up the device addresses of its own device
 * variables (a status word, and the scratch array of the allocation-free entry
 * point) once per device and caches them; a cudaDeviceReset ends the context
 * they belong to, and calls after one are not supported.
 * Kernel choice: the tensor-core kernels run whenever they cover the problem
 * (bf16 inputs, d = 128; prefill C = 64; decode C in {64, 128}), the CUDA-core
 * kernels otherwise.  As a test control, the environment variables
 * HILS_PREFILL_KERNEL=simt and HILS_DECODE_KERNEL=simt force the CUDA-core
 * prefill and decode-attention kernels; results agree within the parity bounds.
 */
#ifndef HILS_H
#define HILS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HILS_API __attribute__((visibility("default")))
#else
#define HILS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define HILS_VERSION 122    /* 1.2.2: adds hils_forward_host (1.2.1: hils_describe; 1.2.0: the backward pass; 1.1.0: window/bias selection and forward, landmarks) */
#define HILS_MAX_K 64       /* largest supported top-k */
#define HILS_MAX_GROUP 16   /* largest supported H / Hkv */

typedef enum {
    HILS_OK = 0,
    HILS_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misaligned pointer */
    HILS_ERR_UNSUPPORTED = 2,   /* valid but not implemented: d, C, k or group size */
    HILS_ERR_CUDA = 3,          /* a CUDA runtime call failed */
    HILS_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up */
    HILS_ERR_WORKSPACE = 5      /* workspace pointer null or smaller than required */
} hils_status;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

typedef struct {
    int B, H, Hkv;        /* batch, query heads, key/value heads (H % Hkv == 0) */
    int N;                /* queries per sequence */
    int T;                /* keys/values per sequence */
    int d;                /* head dimension: 64 or 128 */
    int C;                /* chunk size: 32, 64 or 128 */
    int k;                /* past chunks retrieved per query: 0..HILS_MAX_K */
    int q_offset;         /* position of query 0 */
    hils_dtype in_dtype;  /* Q, K, V, L */
    hils_dtype out_dtype; /* O */
    float scale;          /* logit and retrieval-score scale; 0 selects 1/sqrt(d) */
} hils_problem;

/* Human-readable name of a status code (static string, never NULL). */
HILS_API const char *hils_status_string(int status);

/* Library version, HILS_VERSION of the build. */
HILS_API int hils_version(void);

/* Check a problem description without launching anything. */
HILS_API hils_status hils_validate(const hils_problem *p);

/*
 * The kernels the library would run for problem p with the current test controls, as text:
 * "forward=<k> select=<k> attend=<k>", where forward is "decode-fused" (one cooperative kernel for
 * single-token decode) or "two-call", select is one of "decode-scan", "tc-queries",
 * "tc-heads-resident", "tc-heads", "cuda-cores", and attend is one of "decode-mma", "decode-cuda-cores",
 * "chunk-major", "union-tc", "cuda-cores" (select and attend name what hils_score_select and
 * hils_chunk_attend_fuse run).  Writes at most len bytes including the terminating zero into buf
 * (host memory, owned by the caller); HILS_ERR_INVALID_ARG if buf is NULL or len is too small for the
 * text (at most 80 bytes), the problem's own error if it is invalid.  Launches nothing.
 */
HILS_API hils_status hils_describe(const hils_problem *p, char *buf, size_t len);

/* Workspace bytes each entry point needs for problem p (may be 0). */
HILS_API hils_status hils_score_select_workspace_size(const hils_problem *p, size_t *bytes);
HILS_API hils_status hils_chunk_attend_fuse_workspace_size(const hils_problem *p, size_t *bytes);
HILS_API hils_status hils_forward_workspace_size(const hils_problem *p, size_t *bytes);

/*
 * Steps 1-2 plus the per-head slot scores of step 4 (Sec. 3 "Sparse training";
 * Sec. 4 GQA retrieval).  Reads Q and L; writes sel_idx [B][Hkv][N][k] and
 * sel_score [B][H][N][k+1].  sel_idx may be NULL only when k == 0.
 */
HILS_API hils_status hils_score_select(const hils_problem *p, const void *Q, const void *L,
                              int32_t *sel_idx, float *sel_score,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Steps 3-4 (Abstract; Sec. 3 "Hierarchical softmax") for a given selection:
 * gathers the selected chunks' keys and values once per kv-group, attends
 * inside each, and fuses with softmax(sel_score) per head.  Writes O.
 * sel_idx entries must be -1 or a past chunk of the query (0 <= c < c_i), and
 * a row must not name a chunk twice; the kernels trust this.  With the
 * environment variable HILS_CHECK_SELECTION=1 (a debug aid) the call first
 * checks every row on the GPU, waits for the verdict (synchronising `stream`)
 * and returns HILS_ERR_INVALID_ARG, launching nothing else, when a row breaks
 * the rule.
 * Precision: every product accumulates in float32, and the result is defined
 * for every finite input.  On the bf16 tensor-core prefill kernel the
 * probabilities that multiply V are rounded to 16 bits while V enters exactly:
 * to f16 (relative error 2^-11) for a (b, kv-head) whose values all have
 * magnitude below 65536 (V is converted to f16 in the workspace; values below
 * 2^-14 become f16 subnormals, within 2^-25), and to bf16 (2^-9) otherwise,
 * with V read as given.  The output error from this rounding is at most that
 * relative error times the largest |v| the query attends to.
 */
HILS_API hils_status hils_chunk_attend_fuse(const hils_problem *p, const void *Q, const void *K,
                                   const void *V, const int32_t *sel_idx,
                                   const float *sel_score, void *O,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * The whole forward pass (steps 1-4): hils_score_select then
 * hils_chunk_attend_fuse with the intermediate selection kept in the
 * workspace.  N = 1 runs the single-token decode kernels.
 */
HILS_API hils_status hils_forward(const hils_problem *p, const void *Q, const void *K, const void *V,
                         const void *L, void *O, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * hils_forward on HOST buffers: Q, K, V, L are read from and O is written to host memory (page-locked
 * for the copies to overlap; pageable memory works but serialises them).  The (batch, kv-group) pairs
 * are independent problems [Sec. 4, Architecture: a group's heads share its selection, groups share
 * nothing], so the batch is cut into about eight slices of consecutive pairs; each slice's inputs are
 * copied into one of two device slots on an internal stream, its forward runs on `stream`, and its
 * output is copied back on a second internal stream, so copies in, compute and copies out of
 * different slices overlap.  Layouts as for hils_forward.  The workspace (device memory, owned by
 * the caller, 16-byte aligned) holds the two slots and the slice forward's workspace; its size comes
 * from hils_forward_host_workspace_size.  Stream-ordered: the copies start after the work already
 * queued on `stream`, and work queued on `stream` afterwards (a synchronisation, an event) sees O on
 * the host.  Calls from several host threads are serialised while they enqueue.  Errors: those of
 * hils_forward, HILS_ERR_INVALID_ARG for a NULL host pointer, HILS_ERR_WORKSPACE for a short
 * workspace, HILS_ERR_CUDA if a copy or the internal streams fail (work already queued may then be
 * partly done).  Single-token decode normally keeps its caches on the device and calls hils_forward.
 */
HILS_API hils_status hils_forward_host_workspace_size(const hils_problem *p, size_t *bytes);
HILS_API hils_status hils_forward_host(const hils_problem *p, const void *Q, const void *K, const void *V,
                              const void *L, void *O, void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * Selection with a local window and a per-chunk bias (Sec. 2 Preliminary and
 * Sec. 5 Small-scale Studies, "Experimental setup": a sliding-window branch
 * keeps the recent context in every query's attention; Sec. 3 Methodology,
 * "Linear surrogate for chunk mass": the surrogate mass adds a per-chunk bias
 * to the query-landmark score).  Chunk-aligned reading: the window is the own
 * chunk c_i and the window_chunks - 1 chunks before it (window_chunks >= 1,
 * else HILS_ERR_INVALID_ARG); those are always attended and never retrieval
 * candidates, so retrieval ranks only c <= c_i - window_chunks.  bias
 * [B][Hkv][nL] float, device memory, 4-byte aligned, or NULL (no bias): added
 * to every head's score of chunk c, hence to the group score and to the fusion
 * scores.  Writes the selection in the form hils_chunk_attend_fuse reads for a
 * problem with k' = k + window_chunks - 1 past slots (k' <= HILS_MAX_K, else
 * HILS_ERR_UNSUPPORTED):
 *   sel_idx   [B][Hkv][N][k']   the top-min(k, candidates) chunks in rank order
 *                               (-1 padded to k), then the window's past chunks
 *                               c_i - window_chunks + 1 .. c_i - 1 ascending
 *                               (-1 below chunk 0);
 *   sel_score [B][H][N][k' + 1] each slot's scale * <q_h, L_c> + bias_c, the own
 *                               chunk last, -INFINITY for empty slots.
 * window_chunks = 1 with bias NULL selects what hils_score_select selects.
 * No workspace; Q, L, sel_idx and sel_score as for hils_score_select.
 */
HILS_API hils_status hils_score_select_window(const hils_problem *p, int window_chunks, const float *bias,
                                              const void *Q, const void *L, int32_t *sel_idx, float *sel_score,
                                              void *stream);

/*
 * The windowed, biased forward pass: hils_score_select_window, then
 * hils_chunk_attend_fuse on the problem with k' = k + window_chunks - 1 (the
 * window's chunks are attended and fused like retrieved ones; the own chunk is
 * causal).  The selection is kept in the workspace, whose size
 * hils_forward_window_workspace_size reports.
 */
HILS_API hils_status hils_forward_window_workspace_size(const hils_problem *p, int window_chunks, size_t *bytes);
HILS_API hils_status hils_forward_window(const hils_problem *p, int window_chunks, const float *bias,
                                         const void *Q, const void *K, const void *V, const void *L, void *O,
                                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Landmark generation (Sec. 3 Methodology, "Linear surrogate for chunk mass":
 * a landmark token appended to each chunk supplies a learned query whose
 * attention over the chunk's keys yields the chunk's compressed key).  For
 * every (b, g) and every chunk c in [c_begin, c_end), with key rows
 * t = c*C .. min(c*C + C, T) - 1 and landmark query u_c:
 *   p_t    = softmax over the chunk's rows of scale * <u_c, k_t>
 *   L_c    = sum_t p_t k_t        (in_dtype; bf16 rounded to nearest even)
 *   beta_c = -sum_t p_t ln p_t    (float, the entropy: 0 <= beta_c <= ln rows)
 * Layouts: K [B][Hkv][T][d], U [B][Hkv][nL][d] and L [B][Hkv][nL][d] in
 * in_dtype, beta [B][Hkv][nL] float, nL = ceil(T / C); rows of L and beta
 * outside [c_begin, c_end) are not written.  beta may be NULL (not written).
 * L must not overlap K or U.
 * Uses p->B, Hkv, T, d, C, in_dtype and scale (0 selects 1/sqrt(d)); the
 * other fields are ignored.  Here C may be any chunk size >= 1 (the last
 * chunk may be partial); d is 64 or 128 (else HILS_ERR_UNSUPPORTED).
 * K, U and L 16-byte aligned, beta 4-byte aligned; 0 <= c_begin <= c_end <= nL
 * (else HILS_ERR_INVALID_ARG, nothing launched; c_begin == c_end launches
 * nothing).  A decode step that completes chunk c calls it with
 * c_begin = c, c_end = c + 1.  Reads every key row of the range once; needs
 * no workspace; asynchronous on `stream`.
 */
HILS_API hils_status hils_landmarks(const hils_problem *p, const void *K, const void *U, void *L, float *beta,
                                    int c_begin, int c_end, void *stream);

/*
 * Backward pass through a fixed selection (Sec. 3 Methodology, "Hierarchical
 * softmax": the retrieval scores enter the output as fusion weights, so the
 * loss trains the landmarks and the retrieval through them; a chunk that is
 * not selected gets no gradient; the selection, a discrete choice, is held
 * fixed).  Given the selection sel_idx [B][Hkv][N][k] (as hils_score_select
 * writes it: -1 padded, entries -1 or past chunks of their query, no repeats;
 * the own chunk is implied) and the upstream gradient dO [B][H][N][d]
 * (in_dtype), writes the gradients of sum(O * dO) as float32:
 *   dQ [B][H][N][d], dK and dV [B][Hkv][T][d], dL [B][Hkv][nL][d].
 * With s_c = scale <q, L_c>, w = softmax over the slots of s, P^c the softmax
 * inside chunk c and u_j = <dO, v_j>, per head and query:
 *   dw_c = sum_j P^c_j u_j,  ds_c = w_c (dw_c - sum_c' w_c' dw_c'),
 *   dq   = scale sum_c (ds_c L_c + sum_j dl_j k_j),  dl_j = w_c P^c_j (u_j - dw_c),
 *   dL_c += scale ds_c q,  dk_j += scale dl_j q,  dv_j += w_c P^c_j dO,
 * summed over the queries and heads that reach a row.  Rows of K, V and L that
 * no query reaches get zeros.  The call zeroes dK, dV and dL and accumulates
 * them with float32 atomics (their summation order, hence their last bits,
 * can differ between runs); dQ is written once per row.  Shapes and dtypes as
 * for hils_forward (out_dtype is ignored); every pointer 16-byte aligned.  No
 * workspace; asynchronous on `stream`.  Computed on CUDA cores in float32.
 */
HILS_API hils_status hils_backward(const hils_problem *p, const void *Q, const void *K, const void *V,
                                   const void *L, const int32_t *sel_idx, const void *dO, float *dQ,
                                   float *dK, float *dV, float *dL, void *stream);

/*
 * Synchronise `stream` and report device-side status since the last call:
 * HILS_ERR_TIMEOUT if a bounded wait inside a kernel gave up (the kernel then
 * skipped its remaining work and released its resources), HILS_ERR_CUDA if
 * the synchronisation failed, else HILS_OK.  Clears the recorded status.
 * A recorded timeout is sticky until read here: kernels launched meanwhile
 * give up at their first slow wait, so one failure ends quickly everywhere.
 */
HILS_API hils_status hils_sync_status(void *stream);

/*
 * Debug/test control of the bounded waits: how long (nanoseconds of the GPU's
 * global timer) a kernel waits on a barrier before it records HILS_ERR_TIMEOUT
 * and gives up.  0 restores the default of one second.  Affects kernels
 * launched afterwards; a kernel that gives up still waits for its own copies
 * and MMAs in flight and frees its tensor memory before it exits.
 */
HILS_API hils_status hils_set_wait_limit(long long ns);

/*
 * Test control of the failure path: when `on` is non-zero, tensor-core kernels
 * launched afterwards first wait on a barrier that nothing signals, so that
 * bounded wait expires after the wait limit; the kernel then records
 * HILS_ERR_TIMEOUT, drains and exits.  No GPU fault is involved.  Off by default.
 */
HILS_API hils_status hils_debug_inject_stall(int on);

/*
 * Allocation-free decode selection.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- plugins whose
 * host application owns the whole device memory budget, memory-capped
 * processes that cannot reserve a per-call workspace, and latency-critical
 * paths that must not enter the driver's allocator.
 *
 * Same result as hils_score_select for a single-token decode problem (N == 1),
 * but the kernel's scratch (per-split candidate lists and completion tickets)
 * comes from a fixed array of HILS_NOALLOC_SCRATCH_BYTES in the library's own
 * device memory; the caller still passes Q, L, sel_idx and sel_score.  Every
 * GPU that loads the library holds that array until the process exits.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.
 *   - Problems whose scratch (hils_score_select_workspace_size) exceeds
 *     HILS_NOALLOC_SCRATCH_BYTES return HILS_ERR_WORKSPACE; N != 1 returns
 *     HILS_ERR_UNSUPPORTED.  Nothing is launched in either case.
 *   - The call allocates and frees nothing.  It clears the tickets it needs
 *     before its kernel runs.
 *   - All calls share the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race
 *     and give undefined results.
 */
#define HILS_NOALLOC_SCRATCH_BYTES (1u << 20)   /* 1 MiB per device */
HILS_API hils_status hils_decode_score_select_noalloc(const hils_problem *p, const void *Q, const void *L,
                                                      int32_t *sel_idx, float *sel_score, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H */
