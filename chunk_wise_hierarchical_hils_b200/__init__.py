"""Python binding of libhils.so, the HiLS attention forward library for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/hils.h``.  The functions carry
the C names; tensors may be torch tensors (their data pointers are passed) or
raw integer device addresses.  A missing library raises ImportError: there is
no fallback implementation.

Typical use::

    import chunk_wise_hierarchical_hils_b200 as hils
    p = hils.problem_for(Q, K, C=64, k=16)
    ws = torch.empty(hils.hils_forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    hils.hils_forward(p, Q, K, V, L, O, ws)
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libhils.so")

HILS_OK, HILS_ERR_INVALID_ARG, HILS_ERR_UNSUPPORTED, HILS_ERR_CUDA, HILS_ERR_TIMEOUT, HILS_ERR_WORKSPACE = range(6)
HILS_F32, HILS_BF16 = 0, 1
HILS_MAX_K = 64
HILS_MAX_GROUP = 16

EXPORTS = ("hils_status_string", "hils_version", "hils_validate", "hils_describe", "hils_score_select_workspace_size",
           "hils_chunk_attend_fuse_workspace_size", "hils_forward_workspace_size", "hils_score_select",
           "hils_chunk_attend_fuse", "hils_forward", "hils_forward_host_workspace_size", "hils_forward_host", "hils_sync_status", "hils_set_wait_limit",
           "hils_decode_score_select_noalloc", "hils_debug_inject_stall", "hils_landmarks",
           "hils_score_select_window", "hils_forward_window_workspace_size", "hils_forward_window",
           "hils_backward")
HILS_NOALLOC_SCRATCH_BYTES = 1 << 20


class hils_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("Hkv", ctypes.c_int), ("N", ctypes.c_int),
                ("T", ctypes.c_int), ("d", ctypes.c_int), ("C", ctypes.c_int), ("k", ctypes.c_int),
                ("q_offset", ctypes.c_int), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("scale", ctypes.c_float)]

    def __repr__(self):
        return "hils_problem(%s)" % ", ".join("%s=%r" % (f, getattr(self, f)) for f, _ in self._fields_)


class HilsError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s" % (where, hils_status_string(status)))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libhils.so is not built (expected at %s); run "
                          "`python chunk_wise_hierarchical_hils_b200/build.py`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(hils_problem)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.hils_status_string.argtypes = [ctypes.c_int]
    lib.hils_status_string.restype = ctypes.c_char_p
    lib.hils_version.restype = ctypes.c_int
    lib.hils_validate.argtypes = [P]
    for n in ("hils_score_select_workspace_size", "hils_chunk_attend_fuse_workspace_size",
              "hils_forward_workspace_size"):
        getattr(lib, n).argtypes = [P, ctypes.POINTER(sz)]
    lib.hils_score_select.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
    lib.hils_chunk_attend_fuse.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hils_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hils_forward_host_workspace_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.hils_forward_host.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hils_describe.argtypes = [P, ctypes.c_char_p, sz]
    lib.hils_sync_status.argtypes = [vp]
    lib.hils_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.hils_decode_score_select_noalloc.argtypes = [P, vp, vp, vp, vp, vp]
    lib.hils_debug_inject_stall.argtypes = [ctypes.c_int]
    lib.hils_landmarks.argtypes = [P, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp]
    ci = ctypes.c_int
    lib.hils_score_select_window.argtypes = [P, ci, vp, vp, vp, vp, vp, vp]
    lib.hils_forward_window_workspace_size.argtypes = [P, ci, ctypes.POINTER(sz)]
    lib.hils_forward_window.argtypes = [P, ci, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hils_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    for n in EXPORTS[2:]:
        if n not in ("hils_status_string", "hils_version"):
            getattr(lib, n).restype = ctypes.c_int
    return lib


_lib = _load()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _nbytes(x):
    if x is None:
        return 0
    if isinstance(x, int):
        raise TypeError("pass the workspace size with a raw pointer: (ptr, nbytes)")
    return x.numel() * x.element_size()


def _ws(ws):
    if isinstance(ws, tuple):
        return ws[0], ws[1]
    return _ptr(ws), _nbytes(ws)


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status, where):
    if status != HILS_OK:
        raise HilsError(status, where)


def hils_status_string(status):
    return _lib.hils_status_string(int(status)).decode()


def hils_version():
    return _lib.hils_version()


def hils_describe(p):
    """The kernels the library runs for problem p, e.g. "forward=two-call select=tc-heads-resident
    attend=union-tc" (see include/hils.h)."""
    buf = ctypes.create_string_buffer(128)
    _check(_lib.hils_describe(ctypes.byref(p), buf, ctypes.c_size_t(len(buf))), "hils_describe")
    return buf.value.decode()


def hils_validate(p):
    return _lib.hils_validate(ctypes.byref(p))


def _size(fn, p):
    n = ctypes.c_size_t(0)
    _check(fn(ctypes.byref(p), ctypes.byref(n)), fn.__name__)
    return n.value


def hils_score_select_workspace_size(p):
    return _size(_lib.hils_score_select_workspace_size, p)


def hils_chunk_attend_fuse_workspace_size(p):
    return _size(_lib.hils_chunk_attend_fuse_workspace_size, p)


def hils_forward_workspace_size(p):
    return _size(_lib.hils_forward_workspace_size, p)


def hils_score_select(p, Q, L, sel_idx, sel_score, workspace=None, stream=None):
    wp, wn = _ws(workspace)
    _check(_lib.hils_score_select(ctypes.byref(p), _ptr(Q), _ptr(L), _ptr(sel_idx), _ptr(sel_score), wp, wn,
                                  _stream(stream)), "hils_score_select")


def hils_chunk_attend_fuse(p, Q, K, V, sel_idx, sel_score, O, workspace=None, stream=None):
    wp, wn = _ws(workspace)
    _check(_lib.hils_chunk_attend_fuse(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(sel_idx), _ptr(sel_score),
                                       _ptr(O), wp, wn, _stream(stream)), "hils_chunk_attend_fuse")


def hils_forward(p, Q, K, V, L, O, workspace=None, stream=None):
    wp, wn = _ws(workspace)
    _check(_lib.hils_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(L), _ptr(O), wp, wn,
                             _stream(stream)), "hils_forward")


def hils_forward_host_workspace_size(p):
    return _size(_lib.hils_forward_host_workspace_size, p)


def hils_forward_host(p, Q, K, V, L, O, workspace=None, stream=None):
    """hils_forward on host tensors (page-locked for overlapped copies): Q, K, V, L are read from and O is
    written to host memory, with copies and compute of batch slices overlapped (see include/hils.h)."""
    wp, wn = _ws(workspace)
    _check(_lib.hils_forward_host(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(L), _ptr(O), wp, wn,
                                  _stream(stream)), "hils_forward_host")


def hils_sync_status(stream=None):
    """Returns the status code (HILS_OK or HILS_ERR_TIMEOUT / HILS_ERR_CUDA)."""
    return _lib.hils_sync_status(_stream(stream))


def hils_set_wait_limit(ns):
    """Bounded-wait limit of the kernels in nanoseconds (0 = default, one second)."""
    _check(_lib.hils_set_wait_limit(int(ns)), "hils_set_wait_limit")


def hils_debug_inject_stall(on):
    """Test control: tensor-core kernels wait once on a barrier nothing signals (their bounded wait expires)."""
    _check(_lib.hils_debug_inject_stall(int(bool(on))), "hils_debug_inject_stall")


def hils_decode_score_select_noalloc(p, Q, L, sel_idx, sel_score, stream=None):
    """hils_score_select for N == 1 with the library's fixed scratch: no workspace argument.

    For callers that cannot allocate device memory; see include/hils.h."""
    _check(_lib.hils_decode_score_select_noalloc(ctypes.byref(p), _ptr(Q), _ptr(L), _ptr(sel_idx),
                                                 _ptr(sel_score), _stream(stream)),
           "hils_decode_score_select_noalloc")


def hils_landmarks(p, K, U, L, beta=None, c_begin=0, c_end=None, stream=None):
    """Landmarks L and entropy biases beta of chunks [c_begin, c_end) from keys K and landmark queries U.

    c_end defaults to the number of chunks, ceil(T / C); see include/hils.h."""
    if c_end is None:
        c_end = (p.T + p.C - 1) // p.C
    _check(_lib.hils_landmarks(ctypes.byref(p), _ptr(K), _ptr(U), _ptr(L), _ptr(beta), int(c_begin), int(c_end),
                               _stream(stream)), "hils_landmarks")


def hils_score_select_window(p, window_chunks, bias, Q, L, sel_idx, sel_score, stream=None):
    """Selection with a window of window_chunks chunks and an optional per-chunk bias [B,Hkv,nL] (float32).

    sel_idx holds k + window_chunks - 1 slots per query, sel_score k + window_chunks; see include/hils.h."""
    _check(_lib.hils_score_select_window(ctypes.byref(p), int(window_chunks), _ptr(bias), _ptr(Q), _ptr(L),
                                         _ptr(sel_idx), _ptr(sel_score), _stream(stream)),
           "hils_score_select_window")


def hils_forward_window_workspace_size(p, window_chunks):
    n = ctypes.c_size_t(0)
    _check(_lib.hils_forward_window_workspace_size(ctypes.byref(p), int(window_chunks), ctypes.byref(n)),
           "hils_forward_window_workspace_size")
    return n.value


def hils_forward_window(p, window_chunks, bias, Q, K, V, L, O, workspace=None, stream=None):
    """The forward pass with a local window and a per-chunk bias (bias may be None)."""
    wp, wn = _ws(workspace)
    _check(_lib.hils_forward_window(ctypes.byref(p), int(window_chunks), _ptr(bias), _ptr(Q), _ptr(K), _ptr(V),
                                    _ptr(L), _ptr(O), wp, wn, _stream(stream)), "hils_forward_window")


def hils_backward(p, Q, K, V, L, sel_idx, dO, dQ, dK, dV, dL, stream=None):
    """Gradients dQ, dK, dV, dL (float32 tensors, written) of sum(O * dO) through the selection sel_idx."""
    _check(_lib.hils_backward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(L), _ptr(sel_idx), _ptr(dO), _ptr(dQ),
                              _ptr(dK), _ptr(dV), _ptr(dL), _stream(stream)), "hils_backward")


def problem(B, H, Hkv, N, T, d, C, k, q_offset=0, in_dtype=HILS_BF16, out_dtype=None, scale=0.0):
    return hils_problem(B, H, Hkv, N, T, d, C, k, q_offset, in_dtype,
                        in_dtype if out_dtype is None else out_dtype, float(scale))


def problem_for(Q, K, C, k, q_offset=None, out_dtype=None, scale=0.0):
    """hils_problem from torch tensors Q [B,H,N,d] and K [B,Hkv,T,d].

    q_offset defaults to T - N (the queries are the last N positions)."""
    import torch
    B, H, N, d = Q.shape
    Hkv, T = K.shape[1], K.shape[2]
    dt = {torch.float32: HILS_F32, torch.bfloat16: HILS_BF16}[Q.dtype]
    od = dt if out_dtype is None else {torch.float32: HILS_F32, torch.bfloat16: HILS_BF16}.get(out_dtype, out_dtype)
    return problem(B, H, Hkv, N, T, d, C, k, T - N if q_offset is None else q_offset, dt, od, scale)
