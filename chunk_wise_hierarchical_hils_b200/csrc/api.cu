// api.cu -- the C ABI of libhils.so: validation, workspace sizing, dispatch.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <mutex>

#include "internal.h"
#include "next_rows.h"

namespace hils {

namespace {

__device__ unsigned int g_status;   // device-side status word (one per device)

constexpr long long kDefaultWaitLimit = 1000000000ll;   // ns of the GPU global timer: one second
long long g_wait_limit = kDefaultWaitLimit;
int g_inject_stall = 0;
std::mutex g_mu;

}  // namespace

hils_status device_ctl(DeviceCtl *ctl)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
    static unsigned int *addr[64] = {nullptr};
    if (dev < 0 || dev >= 64) return HILS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!addr[dev]) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_status) != cudaSuccess) return HILS_ERR_CUDA;
        addr[dev] = static_cast<unsigned int *>(a);
    }
    ctl->status = addr[dev];
    ctl->wait_limit = g_wait_limit;
    ctl->inject_stall = g_inject_stall;
    return HILS_OK;
}

namespace {

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

hils_status resolve(const hils_problem *p, Dims *o)
{
    if (!p) return HILS_ERR_INVALID_ARG;
    if (p->B < 1 || p->H < 1 || p->Hkv < 1 || p->N < 1 || p->T < 1 || p->d < 1 || p->C < 1 || p->k < 0)
        return HILS_ERR_INVALID_ARG;
    if (p->H % p->Hkv) return HILS_ERR_INVALID_ARG;
    if (p->q_offset < 0 || (long long)p->q_offset + p->N > p->T) return HILS_ERR_INVALID_ARG;
    if ((p->in_dtype != HILS_F32 && p->in_dtype != HILS_BF16) ||
        (p->out_dtype != HILS_F32 && p->out_dtype != HILS_BF16))
        return HILS_ERR_INVALID_ARG;
    if (!(p->scale >= 0.f) || isinf(p->scale)) return HILS_ERR_INVALID_ARG;
    if (p->d != 64 && p->d != 128) return HILS_ERR_UNSUPPORTED;
    if (p->C != 32 && p->C != 64 && p->C != 128) return HILS_ERR_UNSUPPORTED;
    if (p->k > HILS_MAX_K) return HILS_ERR_UNSUPPORTED;
    const int G = p->H / p->Hkv;
    if (G > HILS_MAX_GROUP) return HILS_ERR_UNSUPPORTED;
    if ((long long)p->B * p->Hkv > 65535 || p->B > 65535) return HILS_ERR_UNSUPPORTED;
    o->B = p->B; o->H = p->H; o->Hkv = p->Hkv; o->G = G;
    o->N = p->N; o->T = p->T; o->d = p->d; o->C = p->C; o->k = p->k;
    o->nL = (p->T + p->C - 1) / p->C;
    o->q_offset = p->q_offset;
    o->scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
    if (o->N == 1 && decode_select_smem_bytes(*o, p->in_dtype) > 200 * 1024) return HILS_ERR_UNSUPPORTED;
    return HILS_OK;
}

namespace {

size_t sel_idx_bytes(const Dims &p) { return align_up((size_t)p.B * p.Hkv * p.N * p.k * sizeof(int32_t), 256); }
size_t sel_score_bytes(const Dims &p) { return align_up((size_t)p.B * p.H * p.N * (p.k + 1) * sizeof(float), 256); }
size_t select_ws(const Dims &p) { return p.N == 1 ? decode_select_ws_bytes(p) : 0; }
// Test control: HILS_PREFILL_ATTEND=union or =chunk forces the tensor-core prefill attention that walks
// each query block's chunk union, or the chunk-major one (where it covers the shape).
int forced_prefill_attend()
{
    const char *force = getenv("HILS_PREFILL_ATTEND");
    if (force && strcmp(force, "union") == 0) return 1;
    if (force && strcmp(force, "chunk") == 0) return 2;
    return 0;
}

bool use_chunk_major(const Dims &p, hils_dtype in)
{
    const char *simt = getenv("HILS_PREFILL_KERNEL");
    if (simt && strcmp(simt, "simt") == 0) return false;
    const int forced = forced_prefill_attend();
    if (forced == 1 || !attend_cm_supported(p, in)) return false;
    return forced == 2 || attend_cm_preferred(p);
}

size_t attend_ws(const Dims &p, hils_dtype in, hils_dtype out)
{
    if (p.N == 1) return decode_attend_ws_bytes(p);
    if (use_chunk_major(p, in)) return attend_cm_ws_bytes(p, out);
    return attend_tc_supported(p, in) ? attend_tc_ws_bytes(p) : 0;
}

// Debug control: HILS_DEBUG=1 prints the CUDA runtime's error string when a launch or runtime call
// of an entry point fails (the status alone says only HILS_ERR_CUDA).
hils_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess) return HILS_OK;
    const char *dbg = getenv("HILS_DEBUG");
    if (dbg && strcmp(dbg, "1") == 0) fprintf(stderr, "hils: CUDA error %d: %s\n", (int)e, cudaGetErrorString(e));
    return HILS_ERR_CUDA;
}

// HILS_PREFILL_KERNEL=simt forces the CUDA-core prefill kernels (used to cross-check the two paths).
bool force_cuda_cores()
{
    const char *force = getenv("HILS_PREFILL_KERNEL");
    return force && strcmp(force, "simt") == 0;
}

// Debug control: HILS_CHECK_SELECTION=1 checks a caller's selection before chunk attention.
bool check_caller_selection()
{
    const char *v = getenv("HILS_CHECK_SELECTION");
    return v && strcmp(v, "1") == 0;
}

// Test control: HILS_SELECT_KERNEL=heads or =queries forces the tensor-core prefill selection with one
// product row per head or per query (where it covers the shape), to cross-check the two.
int forced_select_kernel()
{
    const char *force = getenv("HILS_SELECT_KERNEL");
    if (force && strcmp(force, "heads") == 0) return 1;
    if (force && strcmp(force, "queries") == 0) return 2;
    return 0;
}

// Test control: HILS_PREFILL_KERNEL=persistent runs the union attention as a persistent kernel.
bool persistent_union()
{
    const char *v = getenv("HILS_PREFILL_KERNEL");
    return v && strcmp(v, "persistent") == 0;
}

// Test control: HILS_DECODE_FUSED=0 keeps hils_forward's single-token decode on the two kernels
// (selection, then attention) instead of the fused cooperative kernel.
bool fused_decode_enabled()
{
    const char *v = getenv("HILS_DECODE_FUSED");
    return !(v && strcmp(v, "0") == 0);
}

// Test control: HILS_DECODE_KERNEL=simt keeps decode attention on the CUDA-core kernel.
bool force_decode_cuda_cores()
{
    const char *force = getenv("HILS_DECODE_KERNEL");
    return force && strcmp(force, "simt") == 0;
}

hils_status check_ws(void *ws, size_t have, size_t need)
{
    if (need == 0) return HILS_OK;
    if (!ws || have < need) return HILS_ERR_WORKSPACE;
    if (!aligned16(ws)) return HILS_ERR_INVALID_ARG;
    return HILS_OK;
}

// The selection kernel for a problem (one decision, used by the launch and by hils_describe).
enum class SelKind { DecodeScan, Queries, Heads, CudaCores };

SelKind select_kind(const Dims &p, hils_dtype in)
{
    if (p.N == 1) return SelKind::DecodeScan;
    const int forced = forced_select_kernel();
    if (!force_cuda_cores() && forced != 1 && select_q_supported(p, in) && (forced == 2 || select_q_preferred(p)))
        return SelKind::Queries;
    if (!force_cuda_cores() && select_tc_supported(p, in)) return SelKind::Heads;
    return SelKind::CudaCores;
}

hils_status do_select(const Dims &p, hils_dtype in, const void *Q, const void *L, int32_t *sel_idx,
                      float *sel_score, void *ws, cudaStream_t s)
{
    DeviceCtl ctl;
    hils_status st = device_ctl(&ctl);
    if (st != HILS_OK) return st;
    switch (select_kind(p, in)) {
    case SelKind::DecodeScan: return from_cuda(launch_select_decode(p, in, Q, L, sel_idx, sel_score, ws, ctl, s));
    case SelKind::Queries: return from_cuda(launch_select_prefill_q(p, Q, L, sel_idx, sel_score, ctl, s));
    case SelKind::Heads: return from_cuda(launch_select_prefill_tc(p, Q, L, sel_idx, sel_score, ctl, s));
    default: return from_cuda(launch_select_prefill(p, in, Q, L, sel_idx, sel_score, s));
    }
}

// The attention kernel for a problem (hils_chunk_attend_fuse), likewise.
enum class AttKind { DecodeMma, DecodeCudaCores, ChunkMajor, Union, CudaCores };

AttKind attend_kind(const Dims &p, hils_dtype in)
{
    if (p.N == 1)
        return (!force_decode_cuda_cores() && attend_decode_mma_supported(p, in)) ? AttKind::DecodeMma
                                                                                   : AttKind::DecodeCudaCores;
    if (use_chunk_major(p, in)) return AttKind::ChunkMajor;
    if (!force_cuda_cores() && attend_tc_supported(p, in)) return AttKind::Union;
    return AttKind::CudaCores;
}

// hils_forward's single-token decode runs the fused kernel where it applies.
bool forward_fused(const Dims &p, hils_dtype in)
{
    return p.N == 1 && fused_decode_enabled() && !force_decode_cuda_cores() && decode_fused_supported(p, in);
}

hils_status do_attend(const Dims &p, hils_dtype in, hils_dtype out, const void *Q, const void *K,
                      const void *V, const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                      cudaStream_t s)
{
    DeviceCtl ctl;
    hils_status st = device_ctl(&ctl);
    if (st != HILS_OK) return st;
    switch (attend_kind(p, in)) {
    case AttKind::DecodeMma:
        return from_cuda(launch_attend_decode_mma(p, out, Q, K, V, sel_idx, sel_score, O, ws, ctl, s));
    case AttKind::DecodeCudaCores:
        return from_cuda(launch_attend_decode(p, in, out, Q, K, V, sel_idx, sel_score, O, ws, ctl, s));
    default: return from_cuda(launch_attend_prefill(p, in, out, Q, K, V, sel_idx, sel_score, O, ws, ctl, s));
    }
}

// The problem the chunk attention sees under a window of wc chunks: k + wc - 1 past slots per query.
hils_status resolve_window(const hils_problem *p, int wc, Dims *base, Dims *att)
{
    hils_status st = resolve(p, base);
    if (st != HILS_OK) return st;
    if (wc < 1) return HILS_ERR_INVALID_ARG;
    if ((long long)p->k + wc - 1 > HILS_MAX_K) return HILS_ERR_UNSUPPORTED;
    hils_problem q = *p;
    q.k = p->k + wc - 1;
    return resolve(&q, att);
}

bool aligned4(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

// The windowed, biased selection: prefill on the tensor-core kernel with a row per query where it covers
// the shape, else (decode, float32, other d or k > 32) the CUDA-core kernel.
hils_status select_window(const Dims &p, hils_dtype in, int wc, const float *bias, const void *Q, const void *L,
                          int32_t *sel_idx, float *sel_score, cudaStream_t s)
{
    if (p.N > 1 && !force_cuda_cores() && forced_select_kernel() != 1 && select_q_supported(p, in, wc)) {
        DeviceCtl ctl;
        hils_status st = device_ctl(&ctl);
        if (st != HILS_OK) return st;
        return from_cuda(launch_select_prefill_q(p, Q, L, sel_idx, sel_score, ctl, s, wc, bias));
    }
    return from_cuda(launch_select_window(p, in, wc, bias, Q, L, sel_idx, sel_score, s));
}

}  // namespace

// Prefill dispatch: the tensor-core kernel when it covers the shape, else CUDA cores.
cudaError_t launch_attend_prefill(const Dims &p, hils_dtype in, hils_dtype out, const void *Q, const void *K,
                                  const void *V, const int32_t *sel_idx, const float *sel_score, void *O, void *ws,
                                  const DeviceCtl &ctl, cudaStream_t s)
{
    if (use_chunk_major(p, in))
        return launch_attend_prefill_cm(p, out, Q, K, V, sel_idx, sel_score, O, ws, ctl, s);
    if (!force_cuda_cores() && persistent_union() && attend_tc_persistent_supported(p, in))
        return launch_attend_prefill_tc_persistent(p, out, Q, K, V, sel_idx, sel_score, O, ws, ctl, s);
    if (!force_cuda_cores() && attend_tc_supported(p, in))
        return launch_attend_prefill_tc(p, out, Q, K, V, sel_idx, sel_score, O, ws, ctl, s);
    return launch_attend_prefill_simt(p, in, out, Q, K, V, sel_idx, sel_score, O, s);
}

}  // namespace hils

namespace hils {
namespace {

// ---- forward from host buffers -----------------------------------------------------------------------

constexpr int kHostSlices = 8;   // slices a batch is cut into (fewer when it has fewer units)

struct HostPlan {
    hils_problem slice;                              // the problem of one slice
    int slices;                                      // slices in the batch
    size_t q_bytes, kv_bytes, l_bytes, o_bytes;      // one slice's bytes of Q, K (and V), L, O
    size_t slot_bytes;                               // one device slot: Q, K, V, L, O, each 256-aligned
    size_t fwd_ws;                                   // the slice forward's workspace
};

size_t dtype_bytes(hils_dtype t) { return t == HILS_F32 ? 4 : 2; }

hils_status host_plan(const hils_problem *p, HostPlan *hp)
{
    Dims d;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    // slices of `per` consecutive (b, g) units, each a problem of its own: per divides Hkv (groups
    // g0 .. g0 + per - 1 of one batch element) or is a multiple of Hkv (whole batch elements); the
    // units of a slice are contiguous in every tensor, at offset (first unit) x (bytes per unit)
    const long long units = (long long)d.B * d.Hkv;
    const long long want = (units + kHostSlices - 1) / kHostSlices;
    long long per = units;
    for (long long c = want; c < units; ++c)
        if ((c <= d.Hkv && d.Hkv % c == 0) || (c % d.Hkv == 0 && units % c == 0)) {
            per = c;
            break;
        }
    hils_problem s = *p;
    if (per <= d.Hkv) {
        s.B = 1;
        s.Hkv = (int)per;
        s.H = (int)per * d.G;
    } else {
        s.B = (int)(per / d.Hkv);
    }
    hp->slice = s;
    hp->slices = (int)(units / per);
    const size_t ei = dtype_bytes(p->in_dtype), eo = dtype_bytes(p->out_dtype);
    hp->q_bytes = (size_t)per * d.G * d.N * d.d * ei;
    hp->kv_bytes = (size_t)per * d.T * d.d * ei;
    hp->l_bytes = (size_t)per * d.nL * d.d * ei;
    hp->o_bytes = (size_t)per * d.G * d.N * d.d * eo;
    hp->slot_bytes = align_up(hp->q_bytes, 256) + 2 * align_up(hp->kv_bytes, 256) + align_up(hp->l_bytes, 256) +
                     align_up(hp->o_bytes, 256);
    size_t fw = 0;
    st = hils_forward_workspace_size(&s, &fw);
    if (st != HILS_OK) return st;
    hp->fwd_ws = align_up(fw, 256);
    return HILS_OK;
}

// The internal copy streams and the events of the two slots, per device, created on first use.
struct HostStreams {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
};

std::mutex g_host_mu;   // held while a call enqueues: the events are re-recorded in call order

hils_status host_streams(HostStreams **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
    static HostStreams hs[64];
    if (dev < 0 || dev >= 64) return HILS_ERR_UNSUPPORTED;
    HostStreams &h = hs[dev];
    if (!h.in) {
        bool ok = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&h.start, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&h.end, cudaEventDisableTiming) == cudaSuccess;
        for (int k = 0; k < 2 && ok; ++k)
            ok = cudaEventCreateWithFlags(&h.in_done[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h.comp_done[k], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&h.out_done[k], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            h = HostStreams();   // handles created before the failure stay with the process
            return HILS_ERR_CUDA;
        }
    }
    *out = &h;
    return HILS_OK;
}

}  // namespace
}  // namespace hils

using namespace hils;

extern "C" {

const char *hils_status_string(int status)
{
    switch (status) {
    case HILS_OK: return "HILS_OK";
    case HILS_ERR_INVALID_ARG: return "HILS_ERR_INVALID_ARG: null or misaligned pointer, or invalid shape";
    case HILS_ERR_UNSUPPORTED: return "HILS_ERR_UNSUPPORTED: shape outside the implemented set (d, C, k, group)";
    case HILS_ERR_CUDA: return "HILS_ERR_CUDA: a CUDA runtime call failed";
    case HILS_ERR_TIMEOUT: return "HILS_ERR_TIMEOUT: a bounded device-side wait gave up";
    case HILS_ERR_WORKSPACE: return "HILS_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown hils status";
    }
}

int hils_version(void) { return HILS_VERSION; }

hils_status hils_validate(const hils_problem *p)
{
    Dims d;
    return resolve(p, &d);
}

hils_status hils_describe(const hils_problem *p, char *buf, size_t len)
{
    if (!buf) return HILS_ERR_INVALID_ARG;
    Dims d;
    const hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    const hils_dtype in = p->in_dtype;
    const char *sel = "cuda-cores";
    switch (select_kind(d, in)) {
    case SelKind::DecodeScan: sel = "decode-scan"; break;
    case SelKind::Queries: sel = "tc-queries"; break;
    case SelKind::Heads: sel = select_tc_resident(d) ? "tc-heads-resident" : "tc-heads"; break;
    default: break;
    }
    const char *att = "cuda-cores";
    switch (attend_kind(d, in)) {
    case AttKind::DecodeMma: att = "decode-mma"; break;
    case AttKind::DecodeCudaCores: att = "decode-cuda-cores"; break;
    case AttKind::ChunkMajor: att = "chunk-major"; break;
    case AttKind::Union: att = "union-tc"; break;
    default: break;
    }
    const int n = snprintf(buf, len, "forward=%s select=%s attend=%s", forward_fused(d, in) ? "decode-fused" : "two-call",
                           sel, att);
    if (n < 0 || (size_t)n >= len) {
        if (len) buf[0] = 0;
        return HILS_ERR_INVALID_ARG;
    }
    return HILS_OK;
}

hils_status hils_score_select_workspace_size(const hils_problem *p, size_t *bytes)
{
    Dims d;
    if (!bytes) return HILS_ERR_INVALID_ARG;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    *bytes = select_ws(d);
    return HILS_OK;
}

hils_status hils_chunk_attend_fuse_workspace_size(const hils_problem *p, size_t *bytes)
{
    Dims d;
    if (!bytes) return HILS_ERR_INVALID_ARG;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    *bytes = attend_ws(d, p->in_dtype, p->out_dtype);
    return HILS_OK;
}

hils_status hils_forward_workspace_size(const hils_problem *p, size_t *bytes)
{
    Dims d;
    if (!bytes) return HILS_ERR_INVALID_ARG;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    size_t scratch = select_ws(d) > attend_ws(d, p->in_dtype, p->out_dtype) ? select_ws(d) : attend_ws(d, p->in_dtype, p->out_dtype);
    if (decode_fused_supported(d, p->in_dtype) && decode_fused_ws_bytes(d) > scratch) scratch = decode_fused_ws_bytes(d);
    *bytes = sel_idx_bytes(d) + sel_score_bytes(d) + scratch;
    return HILS_OK;
}

hils_status hils_score_select(const hils_problem *p, const void *Q, const void *L, int32_t *sel_idx,
                              float *sel_score, void *workspace, size_t workspace_bytes, void *stream)
{
    Dims d;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    if (!Q || !L || !sel_score || (d.k > 0 && !sel_idx)) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(L) || (sel_idx && !aligned16(sel_idx)) || !aligned16(sel_score))
        return HILS_ERR_INVALID_ARG;
    st = check_ws(workspace, workspace_bytes, select_ws(d));
    if (st != HILS_OK) return st;
    return do_select(d, p->in_dtype, Q, L, sel_idx, sel_score, workspace, static_cast<cudaStream_t>(stream));
}

hils_status hils_chunk_attend_fuse(const hils_problem *p, const void *Q, const void *K, const void *V,
                                   const int32_t *sel_idx, const float *sel_score, void *O, void *workspace,
                                   size_t workspace_bytes, void *stream)
{
    Dims d;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    if (!Q || !K || !V || !sel_score || !O || (d.k > 0 && !sel_idx)) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(sel_score) ||
        (sel_idx && !aligned16(sel_idx)))
        return HILS_ERR_INVALID_ARG;
    st = check_ws(workspace, workspace_bytes, attend_ws(d, p->in_dtype, p->out_dtype));
    if (st != HILS_OK) return st;
    if (check_caller_selection()) {
        st = check_selection(d, sel_idx, static_cast<cudaStream_t>(stream));
        if (st != HILS_OK) return st;
    }
    return do_attend(d, p->in_dtype, p->out_dtype, Q, K, V, sel_idx, sel_score, O, workspace,
                     static_cast<cudaStream_t>(stream));
}

hils_status hils_forward(const hils_problem *p, const void *Q, const void *K, const void *V, const void *L,
                         void *O, void *workspace, size_t workspace_bytes, void *stream)
{
    Dims d;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    if (!Q || !K || !V || !L || !O) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(L) || !aligned16(O))
        return HILS_ERR_INVALID_ARG;
    size_t need = 0;
    hils_forward_workspace_size(p, &need);
    st = check_ws(workspace, workspace_bytes, need);
    if (st != HILS_OK) return st;
    char *ws = static_cast<char *>(workspace);
    int32_t *sel_idx = reinterpret_cast<int32_t *>(ws);
    float *sel_score = reinterpret_cast<float *>(ws + sel_idx_bytes(d));
    void *scratch = ws + sel_idx_bytes(d) + sel_score_bytes(d);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (forward_fused(d, p->in_dtype)) {
        DeviceCtl ctl;
        st = device_ctl(&ctl);
        if (st != HILS_OK) return st;
        return from_cuda(launch_decode_fused(d, p->out_dtype, Q, K, V, L, sel_idx, sel_score, O, scratch, ctl, s));
    }
    st = do_select(d, p->in_dtype, Q, L, sel_idx, sel_score, scratch, s);
    if (st != HILS_OK) return st;
    return do_attend(d, p->in_dtype, p->out_dtype, Q, K, V, sel_idx, sel_score, O, scratch, s);
}

hils_status hils_forward_host_workspace_size(const hils_problem *p, size_t *bytes)
{
    if (!bytes) return HILS_ERR_INVALID_ARG;
    HostPlan hp;
    const hils_status st = host_plan(p, &hp);
    if (st != HILS_OK) return st;
    *bytes = 2 * hp.slot_bytes + hp.fwd_ws;
    return HILS_OK;
}

hils_status hils_forward_host(const hils_problem *p, const void *Q, const void *K, const void *V, const void *L,
                              void *O, void *workspace, size_t workspace_bytes, void *stream)
{
    HostPlan hp;
    hils_status st = host_plan(p, &hp);
    if (st != HILS_OK) return st;
    if (!Q || !K || !V || !L || !O) return HILS_ERR_INVALID_ARG;
    st = check_ws(workspace, workspace_bytes, 2 * hp.slot_bytes + hp.fwd_ws);
    if (st != HILS_OK) return st;
    std::lock_guard<std::mutex> lk(g_host_mu);
    HostStreams *h = nullptr;
    st = host_streams(&h);
    if (st != HILS_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    void *fws = ws + 2 * hp.slot_bytes;
    const char *qh = static_cast<const char *>(Q), *kh = static_cast<const char *>(K);
    const char *vh = static_cast<const char *>(V), *lh = static_cast<const char *>(L);
    char *oh = static_cast<char *>(O);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    if (!ok(cudaEventRecord(h->start, s)) || !ok(cudaStreamWaitEvent(h->in, h->start, 0)) ||
        !ok(cudaStreamWaitEvent(h->out, h->start, 0)))
        return HILS_ERR_CUDA;
    for (int i = 0; i < hp.slices; ++i) {
        const int k = i & 1;
        char *dq = ws + (size_t)k * hp.slot_bytes;
        char *dk = dq + align_up(hp.q_bytes, 256);
        char *dv = dk + align_up(hp.kv_bytes, 256);
        char *dl = dv + align_up(hp.kv_bytes, 256);
        char *dout = dl + align_up(hp.l_bytes, 256);
        // copies in: after slice i - 2's forward has read this slot
        if (i >= 2 && !ok(cudaStreamWaitEvent(h->in, h->comp_done[k], 0))) return HILS_ERR_CUDA;
        if (!ok(cudaMemcpyAsync(dq, qh + (size_t)i * hp.q_bytes, hp.q_bytes, cudaMemcpyHostToDevice, h->in)) ||
            !ok(cudaMemcpyAsync(dk, kh + (size_t)i * hp.kv_bytes, hp.kv_bytes, cudaMemcpyHostToDevice, h->in)) ||
            !ok(cudaMemcpyAsync(dv, vh + (size_t)i * hp.kv_bytes, hp.kv_bytes, cudaMemcpyHostToDevice, h->in)) ||
            !ok(cudaMemcpyAsync(dl, lh + (size_t)i * hp.l_bytes, hp.l_bytes, cudaMemcpyHostToDevice, h->in)) ||
            !ok(cudaEventRecord(h->in_done[k], h->in)))
            return HILS_ERR_CUDA;
        // the forward: after its inputs landed and slice i - 2's output left this slot
        if (!ok(cudaStreamWaitEvent(s, h->in_done[k], 0))) return HILS_ERR_CUDA;
        if (i >= 2 && !ok(cudaStreamWaitEvent(s, h->out_done[k], 0))) return HILS_ERR_CUDA;
        st = hils_forward(&hp.slice, dq, dk, dv, dl, dout, fws, hp.fwd_ws, stream);
        if (st != HILS_OK) return st;
        if (!ok(cudaEventRecord(h->comp_done[k], s))) return HILS_ERR_CUDA;
        // copy out
        if (!ok(cudaStreamWaitEvent(h->out, h->comp_done[k], 0)) ||
            !ok(cudaMemcpyAsync(oh + (size_t)i * hp.o_bytes, dout, hp.o_bytes, cudaMemcpyDeviceToHost, h->out)) ||
            !ok(cudaEventRecord(h->out_done[k], h->out)))
            return HILS_ERR_CUDA;
    }
    // the caller's stream continues once the last output copy is done (the copy stream runs in order)
    if (!ok(cudaEventRecord(h->end, h->out)) || !ok(cudaStreamWaitEvent(s, h->end, 0))) return HILS_ERR_CUDA;
    return HILS_OK;
}

hils_status hils_score_select_window(const hils_problem *p, int window_chunks, const float *bias, const void *Q,
                                     const void *L, int32_t *sel_idx, float *sel_score, void *stream)
{
    Dims d, da;
    hils_status st = resolve_window(p, window_chunks, &d, &da);
    if (st != HILS_OK) return st;
    if (!Q || !L || !sel_score || (da.k > 0 && !sel_idx)) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(L) || (sel_idx && !aligned16(sel_idx)) || !aligned16(sel_score) ||
        !aligned4(bias))
        return HILS_ERR_INVALID_ARG;
    return select_window(d, p->in_dtype, window_chunks, bias, Q, L, sel_idx, sel_score,
                         static_cast<cudaStream_t>(stream));
}

hils_status hils_forward_window_workspace_size(const hils_problem *p, int window_chunks, size_t *bytes)
{
    Dims d, da;
    if (!bytes) return HILS_ERR_INVALID_ARG;
    hils_status st = resolve_window(p, window_chunks, &d, &da);
    if (st != HILS_OK) return st;
    *bytes = sel_idx_bytes(da) + sel_score_bytes(da) + attend_ws(da, p->in_dtype, p->out_dtype);
    return HILS_OK;
}

hils_status hils_forward_window(const hils_problem *p, int window_chunks, const float *bias, const void *Q,
                                const void *K, const void *V, const void *L, void *O, void *workspace,
                                size_t workspace_bytes, void *stream)
{
    Dims d, da;
    hils_status st = resolve_window(p, window_chunks, &d, &da);
    if (st != HILS_OK) return st;
    if (!Q || !K || !V || !L || !O) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(L) || !aligned16(O) || !aligned4(bias))
        return HILS_ERR_INVALID_ARG;
    const size_t need = sel_idx_bytes(da) + sel_score_bytes(da) + attend_ws(da, p->in_dtype, p->out_dtype);
    st = check_ws(workspace, workspace_bytes, need);
    if (st != HILS_OK) return st;
    char *ws = static_cast<char *>(workspace);
    int32_t *sel_idx = reinterpret_cast<int32_t *>(ws);
    float *sel_score = reinterpret_cast<float *>(ws + sel_idx_bytes(da));
    void *scratch = ws + sel_idx_bytes(da) + sel_score_bytes(da);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = select_window(d, p->in_dtype, window_chunks, bias, Q, L, sel_idx, sel_score, s);
    if (st != HILS_OK) return st;
    return do_attend(da, p->in_dtype, p->out_dtype, Q, K, V, sel_idx, sel_score, O, scratch, s);
}

hils_status hils_landmarks(const hils_problem *p, const void *K, const void *U, void *L, float *beta, int c_begin,
                           int c_end, void *stream)
{
    if (!p) return HILS_ERR_INVALID_ARG;
    if (p->B < 1 || p->Hkv < 1 || p->T < 1 || p->C < 1) return HILS_ERR_INVALID_ARG;
    if (p->in_dtype != HILS_F32 && p->in_dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
    if (!(p->scale >= 0.f) || isinf(p->scale)) return HILS_ERR_INVALID_ARG;
    if (p->d != 64 && p->d != 128) return HILS_ERR_UNSUPPORTED;
    const long long nL = ((long long)p->T + p->C - 1) / p->C;
    if (c_begin < 0 || c_end < c_begin || c_end > nL) return HILS_ERR_INVALID_ARG;
    if (!K || !U || !L) return HILS_ERR_INVALID_ARG;
    if (!aligned16(K) || !aligned16(U) || !aligned16(L) || (reinterpret_cast<uintptr_t>(beta) & 3u))
        return HILS_ERR_INVALID_ARG;
    if (!landmarks_launchable(p->B, p->Hkv, c_end - c_begin)) return HILS_ERR_UNSUPPORTED;
    const float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
    return from_cuda(launch_landmarks(p->B, p->Hkv, p->T, p->d, p->C, scale, p->in_dtype, K, U, L, beta, c_begin,
                                      c_end, static_cast<cudaStream_t>(stream)));
}

hils_status hils_backward(const hils_problem *p, const void *Q, const void *K, const void *V, const void *L,
                          const int32_t *sel_idx, const void *dO, float *dQ, float *dK, float *dV, float *dL,
                          void *stream)
{
    Dims d;
    hils_status st = resolve(p, &d);
    if (st != HILS_OK) return st;
    if (!Q || !K || !V || !L || !dO || !dQ || !dK || !dV || !dL || (d.k > 0 && !sel_idx)) return HILS_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(L) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV) || !aligned16(dL) || (sel_idx && !aligned16(sel_idx)))
        return HILS_ERR_INVALID_ARG;
    if (backward_smem_bytes(d) > 227 * 1024) return HILS_ERR_UNSUPPORTED;
    if ((long long)d.B * d.Hkv * d.N > 0x7FFFFFFFll) return HILS_ERR_UNSUPPORTED;
    return from_cuda(launch_backward(d, p->in_dtype, Q, K, V, L, sel_idx, dO, dQ, dK, dV, dL,
                                     static_cast<cudaStream_t>(stream)));
}

hils_status hils_sync_status(void *stream)
{
    DeviceCtl ctl;
    hils_status st = device_ctl(&ctl);
    if (st != HILS_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HILS_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, ctl.status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return HILS_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpy(ctl.status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return HILS_ERR_CUDA;
        return HILS_ERR_TIMEOUT;
    }
    return HILS_OK;
}

hils_status hils_set_wait_limit(long long ns)
{
    if (ns < 0) return HILS_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    g_wait_limit = ns == 0 ? kDefaultWaitLimit : ns;
    return HILS_OK;
}

hils_status hils_debug_inject_stall(int on)
{
    std::lock_guard<std::mutex> lk(g_mu);
    g_inject_stall = on ? 1 : 0;
    return HILS_OK;
}

}  // extern "C"
