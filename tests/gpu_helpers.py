"""Shared helpers of the GPU tests: hand-built operands and comparisons."""
import numpy as np
import torch

import sparse_activation_quantization_b200 as sq
from oracle.formats import e2m1_decode, e4m3_decode
from tests import _layout


def ensure_built():
    from sparse_activation_quantization_b200 import build
    build.build()
    sq.lib()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), f"needs sm_100, got sm_{major}{minor}"


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(x_f32):
    """float32 numpy array holding bf16 values -> bf16 CUDA tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32)).to(torch.bfloat16).cuda()


def act_from_logical(T, K, mode, r_codes, r_sf, sp_codes=None, meta=None, sp_sf=None, s_g=1.0):
    """PreparedAct whose buffers hold hand-built logical operands.  The tile
    padding rows past T hold random bytes (invalid metadata, NaN-coded scales
    included): sharq_linear must not depend on them."""
    act = sq.PreparedAct(T, K, mode)
    Tp = act.view.Tp
    g = np.random.default_rng(99)
    junk = lambda a: np.concatenate([a, g.integers(0, 256 if a.dtype == np.uint8 else 16,
                                                   (Tp - T, *a.shape[1:])).astype(a.dtype)])
    act.buf.zero_()
    nib = lambda a: np.concatenate([a, g.integers(0, 16, (Tp - T, *a.shape[1:])).astype(np.uint8)])
    rc = _layout.tile_codes(nib(r_codes))
    act.region("r_codes", rc.size).copy_(to_dev(rc))
    rs = _layout.tile_sf(junk(r_sf), 16)
    act.region("r_sf", rs.size).copy_(to_dev(rs))
    if mode == sq.SHARQ_MODE_SHARQ:
        sc = _layout.tile_sp_codes(nib(sp_codes))
        act.region("sp_codes", sc.size).copy_(to_dev(sc))
        mt = _layout.tile_meta(nib(meta))
        act.region("meta", mt.size).copy_(to_dev(mt))
        ss = _layout.tile_sf(junk(sp_sf), 32)
        act.region("sp_sf", ss.size).copy_(to_dev(ss))
    act.region("s_g", 4).view(torch.float32).fill_(float(s_g))
    return act


class RawWeight:
    """Packed-weight buffer filled from hand-built logical codes / scales."""

    def __init__(self, codes, sf32, s_w=1.0):
        E, D, K = codes.shape
        self.K, self.D, self.E = K, D, E
        n = sq.sharq_weight_bytes(K, D, E)
        self.buf = torch.zeros(n, dtype=torch.uint8, device="cuda")
        self.view = sq.sharq_weight_view(self.buf.data_ptr(), K, D, E)
        base = self.buf.data_ptr()

        def put(ptr, arr):
            off = ptr - base
            self.buf[off:off + arr.size].copy_(to_dev(arr))
        put(self.view.codes, np.concatenate([_layout.tile_codes(codes[e]) for e in range(E)]))
        put(self.view.sf32, np.concatenate([_layout.tile_sf(sf32[e], 32) for e in range(E)]))
        sf16 = np.repeat(sf32, 2, axis=-1)
        put(self.view.sf16, np.concatenate([_layout.tile_sf(sf16[e], 16) for e in range(E)]))
        sw = np.full(E, s_w, dtype=np.float32) if np.isscalar(s_w) else np.asarray(s_w, np.float32)
        put(self.view.s_w, sw.view(np.uint8))


def dequant_sparse_logical(sp_codes, meta, sp_sf):
    """[T, K] float64 activation of the sparse operand from logical arrays."""
    T, Kh = sp_codes.shape
    K = 2 * Kh
    vals = (e2m1_decode(sp_codes).reshape(T, K // 32, 16) * e4m3_decode(sp_sf)[..., None]).reshape(T, K // 8, 4)
    lo, hi = (meta & 3).astype(int), (meta >> 2).astype(int)
    out = np.zeros((T, K // 8, 8))
    rows = np.arange(T)[:, None]
    cols = np.arange(K // 8)[None, :]
    out[rows, cols, 2 * lo] = vals[..., 0]
    out[rows, cols, 2 * lo + 1] = vals[..., 1]
    out[rows, cols, 2 * hi] = vals[..., 2]
    out[rows, cols, 2 * hi + 1] = vals[..., 3]
    return out.reshape(T, K)


def dequant_dense_logical(codes, sf, per):
    R, K = codes.shape
    return (e2m1_decode(codes).reshape(R, K // per, per) * e4m3_decode(sf)[..., None]).reshape(R, K)


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)


def random_meta(g, shape):
    """valid 4:8 in-pairs nibbles p_lo | p_hi << 2 with p_lo < p_hi"""
    pairs = np.array([lo | (hi << 2) for lo in range(4) for hi in range(lo + 1, 4)], dtype=np.uint8)
    return pairs[g.integers(0, len(pairs), shape)]
