"""sharq_linear on hand-built operands vs a float64 numpy product (GPU).

The operands are random codes, scale bytes and metadata written directly in
the tiled layout of include/sharq.h, so these tests pin the MMA data layout
(nibble order, swizzles, scale-factor atoms, metadata nibbles) independently
of sharq_prep.  Scale bytes are powers of two and global scales are 1, so
every product and partial sum is exact in float32 and the GEMM must match to
float32 accumulation error.
"""
import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

POW2_E4M3 = np.array([0x30, 0x38, 0x40, 0x48], dtype=np.uint8)   # 0.5, 1, 2, 4


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def _operands(seed, T, K, D, E=1):
    g = np.random.default_rng(seed)
    r_codes = g.integers(0, 16, (T, K)).astype(np.uint8)
    r_sf = POW2_E4M3[g.integers(0, 4, (T, K // 16))]
    sp_codes = g.integers(0, 16, (T, K // 2)).astype(np.uint8)
    meta = H.random_meta(g, (T, K // 8))
    sp_sf = POW2_E4M3[g.integers(0, 4, (T, K // 32))]
    w_codes = g.integers(0, 16, (E, D, K)).astype(np.uint8)
    w_sf32 = POW2_E4M3[g.integers(0, 4, (E, D, K // 32))]
    return r_codes, r_sf, sp_codes, meta, sp_sf, w_codes, w_sf32


def _run(act, w, T, D, out_f32=True, offsets=None):
    y = sq.linear(act, w, out_dtype=torch.float32 if out_f32 else torch.bfloat16,
                  group_offsets=offsets)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


@pytest.mark.parametrize("T,K,D", [(128, 256, 256), (200, 512, 384), (16, 768, 128), (1, 256, 512)])
def test_dense_nvfp4_mma_exact(T, K, D):
    r_codes, r_sf, _, _, _, w_codes, w_sf32 = _operands(1, T, K, D)
    act = H.act_from_logical(T, K, sq.SHARQ_MODE_NVFP4, r_codes, r_sf)
    w = H.RawWeight(w_codes, w_sf32)
    y = _run(act, w, T, D)
    a = H.dequant_dense_logical(r_codes, r_sf, 16)
    b = H.dequant_dense_logical(w_codes[0], np.repeat(w_sf32[0], 2, -1), 16)
    ref = a @ b.T
    assert H.rel_fro(y, ref) < 1e-6, H.rel_fro(y, ref)


@pytest.mark.parametrize("T,K,D", [(128, 256, 256), (200, 512, 384), (16, 768, 128)])
def test_sparse_mma_exact(T, K, D):
    """SHARQ mode with a zero residual: only the sparse MMA contributes."""
    _, _, sp_codes, meta, sp_sf, w_codes, w_sf32 = _operands(2, T, K, D)
    zero_c = np.zeros((T, K), np.uint8)
    zero_s = np.zeros((T, K // 16), np.uint8)
    act = H.act_from_logical(T, K, sq.SHARQ_MODE_SHARQ, zero_c, zero_s, sp_codes, meta, sp_sf)
    w = H.RawWeight(w_codes, w_sf32)
    y = _run(act, w, T, D)
    a = H.dequant_sparse_logical(sp_codes, meta, sp_sf)
    b = H.dequant_dense_logical(w_codes[0], w_sf32[0], 32)
    ref = a @ b.T
    assert H.rel_fro(y, ref) < 1e-6, H.rel_fro(y, ref)


@pytest.mark.parametrize("T,K,D", [(128, 256, 256), (257, 1024, 640)])
def test_dual_path_single_accumulator(T, K, D):
    r_codes, r_sf, sp_codes, meta, sp_sf, w_codes, w_sf32 = _operands(3, T, K, D)
    act = H.act_from_logical(T, K, sq.SHARQ_MODE_SHARQ, r_codes, r_sf, sp_codes, meta, sp_sf,
                             s_g=0.375)
    w = H.RawWeight(w_codes, w_sf32, s_w=0.0625)
    y = _run(act, w, T, D)
    a = H.dequant_sparse_logical(sp_codes, meta, sp_sf) + H.dequant_dense_logical(r_codes, r_sf, 16)
    b = H.dequant_dense_logical(w_codes[0], w_sf32[0], 32)
    ref = (a @ b.T) * (0.375 * 0.0625)
    assert H.rel_fro(y, ref) < 1e-6, H.rel_fro(y, ref)
    yb = _run(act, w, T, D, out_f32=False)
    bf = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(yb, bf) or H.rel_fro(yb, bf) < 1e-3


def test_grouped_experts():
    K, D, E = 512, 256, 4
    offs = np.array([0, 128, 128, 384, 512], dtype=np.int32)
    T = int(offs[-1])
    r_codes, r_sf, sp_codes, meta, sp_sf, w_codes, w_sf32 = _operands(4, T, K, D, E)
    act = H.act_from_logical(T, K, sq.SHARQ_MODE_SHARQ, r_codes, r_sf, sp_codes, meta, sp_sf)
    sw = np.array([1.0, 2.0, 0.5, 0.25], np.float32)
    w = H.RawWeight(w_codes, w_sf32, s_w=sw)
    y = _run(act, w, T, D, offsets=torch.from_numpy(offs).cuda())
    a = H.dequant_sparse_logical(sp_codes, meta, sp_sf) + H.dequant_dense_logical(r_codes, r_sf, 16)
    for e in range(E):
        lo, hi = offs[e], offs[e + 1]
        if hi == lo:
            continue
        b = H.dequant_dense_logical(w_codes[e], w_sf32[e], 32)
        ref = (a[lo:hi] @ b.T) * sw[e]
        assert H.rel_fro(y[lo:hi], ref) < 1e-6, (e, H.rel_fro(y[lo:hi], ref))
