"""Device-side input generation (ctypes wrapper of synth/gen_cuda.cu).

Produces the same values as :mod:`synth.workloads`, whole tensors at a time, for
workloads too large to generate on the host.  Test and benchmark infrastructure.
"""
import ctypes
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen_cuda.cu")
_LIB = os.path.join(_HERE, "_build", "libsynth.so")
_lib = None


class synth_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("Hkv", ctypes.c_int), ("N", ctypes.c_int),
                ("T", ctypes.c_int), ("d", ctypes.c_int), ("C", ctypes.c_int), ("q_offset", ctypes.c_int),
                ("dtype", ctypes.c_int), ("seed", ctypes.c_ulonglong), ("input_scale", ctypes.c_int),
                ("l_mode", ctypes.c_int), ("l_noise", ctypes.c_double), ("n_needles", ctypes.c_int),
                ("needle_period", ctypes.c_int), ("needle_shift", ctypes.c_double)]


def build(force=False):
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + ".tmp%d" % os.getpid()
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                           "-fmad=false", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared", "-o", tmp, _SRC])
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.synth_fill.argtypes = [ctypes.POINTER(synth_params)] + [ctypes.c_void_p] * 4
        _lib.synth_fill.restype = ctypes.c_int
    return _lib


def params(w):
    return synth_params(w.B, w.H, w.Hkv, w.N, w.T, w.d, w.C, w.q_offset, 0 if w.dtype == "f32" else 1, w.seed,
                        int(w.input_scale), 1 if w.l_mode == "chunkmean" else 0, w.l_noise, w.n_needles,
                        w.needle_period if w.needle_period else 1, w.needle_shift)


def _p(t):
    return None if t is None else t.data_ptr()


def fill(w, Q=None, K=None, V=None, L=None):
    """Fill the given torch CUDA tensors with workload w's inputs (synchronous)."""
    p = params(w)
    rc = lib().synth_fill(ctypes.byref(p), _p(Q), _p(K), _p(V), _p(L))
    if rc != 0:
        raise RuntimeError("synth_fill failed with cudaError %d" % rc)


def alloc_inputs(w, device="cuda"):
    """Allocate and fill Q, K, V, L on the device; returns a dict of torch tensors."""
    import torch
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    Q = torch.empty((w.B, w.H, w.N, w.d), dtype=dt, device=device)
    K = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=dt, device=device)
    V = torch.empty_like(K)
    L = torch.empty((w.B, w.Hkv, w.nL, w.d), dtype=dt, device=device)
    fill(w, Q, K, V, L)
    return {"Q": Q, "K": K, "V": V, "L": L}
