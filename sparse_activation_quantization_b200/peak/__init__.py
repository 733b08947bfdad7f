"""Measured FP4 tensor-core peaks of the current GPU (roofline denominators).

Runs the tcgen05 microbenchmark in ``fp4_peak.cu`` (built next to it as
``libsharq_peak.so`` by the package build) on every SM: back-to-back dense
``kind::mxf4nvf4`` block16 MMAs, or 4:8-sparse ones, 128 x N from shared
memory into TMEM.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "libsharq_peak.so")


def fp4_peaks(n256=True, iters=400):
    """{'dense_pflops', 'sparse_pflops', 'effective_pflops'} for N = 256 (or
    128) tiles; sparse counts logical FLOPs; effective is the rate of the
    dual GEMM's 2TKD when both paths run at their peaks."""
    L = ctypes.CDLL(LIB)
    f = L.sharq_fp4_peak
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                  ctypes.POINTER(ctypes.c_double)]
    out = {}
    for name, sp in (("dense", 0), ("sparse", 1)):
        r, ns = ctypes.c_double(), ctypes.c_double()
        if f(sp, 1 if n256 else 0, iters, ctypes.byref(r), ctypes.byref(ns)) != 0:
            raise RuntimeError("fp4 peak microbenchmark failed")
        out[f"{name}_pflops"] = r.value / 1e15
    # a dual GEMM does 2TKD logical FLOPs on each path; its effective rate
    # (2TKD over the time of both) is the harmonic combination
    out["effective_pflops"] = 1.0 / (1.0 / out["dense_pflops"] + 1.0 / out["sparse_pflops"])
    out["n"] = 256 if n256 else 128
    return out
