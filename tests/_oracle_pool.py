"""Oracle-side workers of the full-size parity tests.

These functions run in a pool of processes started with the ``spawn`` method
(never forked from a process that has touched the GPU).  They import numpy
and the oracle only.  Each one prepares a chunk of rows with the oracle,
given the whole tensor's per-tensor scale, and returns the prepared operands
together with the oracle's float64 product of those rows with a set of
dequantized weight columns.
"""
import multiprocessing as mp
import os

import numpy as np

from oracle import sharq as O

_POOL = None


def pool():
    """The shared spawn pool (created once per test process)."""
    global _POOL
    if _POOL is None:
        n = max(1, min(16, len(os.sched_getaffinity(0))))
        _POOL = mp.get_context("spawn").Pool(n)
    return _POOL


def row_stats(args):
    """max |Xn| over a chunk of rows (the per-tensor scale's input)."""
    x, gamma, eps = args
    xn, _ = O.rmsnorm(x, gamma, eps)
    return np.float32(np.max(np.abs(xn))) if xn.size else np.float32(0)


def prep_rows(args):
    """Prepared operands of a chunk of rows under the tensor's scale s_g, and
    y = (X~_sp + R~) W~ * s_g * s_w for each weight's sampled columns."""
    x, gamma, eps, s_g, weights = args
    p = O.prep(x, gamma, eps, s_g=s_g)
    out = {k: p[k] for k in ("meta", "sp_codes", "sp_sf", "r_codes", "r_sf")}
    if weights:
        a = O.dequant_sparse(p) + O.dequant_residual(p)
        out["y"] = [(a @ wt) * (np.float64(s_g) * np.float64(s_w)) for wt, s_w in weights]
    return out


def tensor_scale(x, gamma, eps, chunk):
    """The oracle's per-tensor scale of x, from row chunks in parallel."""
    parts = pool().map(row_stats, [(x[i:i + chunk], gamma, eps) for i in range(0, len(x), chunk)])
    gmax = np.float32(max(parts)) if parts else np.float32(0)
    return np.float32(1.0) if gmax == 0 else np.float32(gmax / O.GLOBAL_DIV)


def sampled_weight(w, cols):
    """(dequantized columns W~[:, cols] in float64 without s_w, s_w): the
    columns quantize exactly as the whole weight's pack does, since NVFP4
    scales run per output column and s_w is the whole weight's amax."""
    from oracle.formats import e2m1_decode, e4m3_decode
    amax = np.float32(np.max(np.abs(w)))
    s_w = np.float32(1.0) if amax == 0 else np.float32(amax / O.GLOBAL_DIV)
    codes, sb, _ = O.nvfp4_quant(np.ascontiguousarray(w[:, cols].T).reshape(len(cols), -1, 32), s_w)
    wt = (e2m1_decode(codes) * e4m3_decode(sb)[..., None]).reshape(len(cols), -1).T
    return np.ascontiguousarray(wt), s_w


def prep_all(x, gamma, eps, s_g, weights, chunk):
    """prep_rows over every chunk of x (in parallel), concatenated."""
    res = pool().map(prep_rows, [(x[i:i + chunk], gamma, eps, s_g, weights) for i in range(0, len(x), chunk)])
    out = {k: np.concatenate([r[k] for r in res]) for k in ("meta", "sp_codes", "sp_sf", "r_codes", "r_sf")}
    if weights:
        out["y"] = [np.concatenate([r["y"][j] for r in res]) for j in range(len(weights))]
    return out
