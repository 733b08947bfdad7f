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


def _peak(fn, *args):
    r, ns = ctypes.c_double(), ctypes.c_double()
    if fn(*args, ctypes.byref(r), ctypes.byref(ns)) != 0:
        raise RuntimeError("fp4 peak microbenchmark failed")
    return r.value / 1e15


def fp4_peaks(n256=True, iters=400):
    """Measured FP4 tensor peaks in PFLOP/s (sparse counts logical FLOPs):
    one CTA per SM issuing 128 x N MMAs (N = 256, or 128), and CTA pairs
    issuing the cta_group::2 256 x 256 MMAs of the prefill GEMM.  The
    'dense_pflops' and 'sparse_pflops' entries are the better of the two
    forms; 'effective_pflops' is the rate of the dual GEMM's 2TKD when both
    paths run at those peaks (their harmonic combination)."""
    L = ctypes.CDLL(LIB)
    f1 = L.sharq_fp4_peak
    f1.restype = ctypes.c_int
    f1.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                   ctypes.POINTER(ctypes.c_double)]
    f2 = L.sharq_fp4_peak_pair
    f2.restype = ctypes.c_int
    f2.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
    out = {"n": 256 if n256 else 128}
    for name, sp in (("dense", 0), ("sparse", 1)):
        one = _peak(f1, sp, 1 if n256 else 0, iters)
        pair = _peak(f2, sp, iters)
        out[f"{name}_pflops_1cta"] = one
        out[f"{name}_pflops_pair"] = pair
        out[f"{name}_pflops"] = max(one, pair)
    # a dual GEMM does 2TKD logical FLOPs on each path; its effective rate
    # (2TKD over the time of both) is the harmonic combination
    out["effective_pflops"] = 1.0 / (1.0 / out["dense_pflops"] + 1.0 / out["sparse_pflops"])
    return out
