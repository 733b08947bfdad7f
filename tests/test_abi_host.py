"""Host-side checks of the C ABI (CPU only, no compute calls).

The library must load, export every function include/sharq.h declares, and
answer its pure host queries (sizes, views, argument checks) correctly.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import sparse_activation_quantization_b200 as sq
from tests import _layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from sparse_activation_quantization_b200 import build
    build.build()
    return sq.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "sharq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sharq_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(sq.EXPORTED_SYMBOLS)
    assert sq.sharq_abi_version() == 2


def test_sizes(L):
    T, K, D = 130, 512, 384
    Tp = 256
    tiles = (Tp // 128) * (K // 256)
    a = sq.sharq_act_bytes(T, K, sq.SHARQ_MODE_SHARQ)
    assert a >= tiles * (16384 + 2048 + 8192 + 2048 + 1024) + Tp * 4
    n = sq.sharq_act_bytes(T, K, sq.SHARQ_MODE_NVFP4)
    assert tiles * (16384 + 2048) + Tp * 4 <= n < a
    w = sq.sharq_weight_bytes(K, D, 2)
    assert w >= 2 * (D // 128) * (K // 256) * (16384 + 1024 + 2048) + 8
    # 0.59375 bytes per weight element: 0.5 codes + 1/32 + 1/16 scales
    assert abs(sq.sharq_weight_bytes(4096, 4096, 1) / (4096 * 4096) - 0.59375) < 1e-3
    # bad shapes -> 0
    assert sq.sharq_act_bytes(16, 200, 0) == 0
    assert sq.sharq_weight_bytes(256, 100, 1) == 0
    assert sq.sharq_act_bytes(-1, 256, 0) == 0
    assert sq.sharq_act_bytes(16, 256, 99) == 0
    # MXFP4: E8M0 scales per 64 K (sparse view) and per 32 K (dense view)
    assert abs(sq.sharq_weight_bytes_fmt(4096, 4096, 1, sq.SHARQ_FMT_MXFP4) / (4096 * 4096) - 0.546875) < 1e-3
    assert sq.sharq_weight_bytes_fmt(4096, 4096, 1, 7) == 0
    mx = sq.sharq_act_bytes(T, K, sq.SHARQ_MODE_MXFP4)
    assert mx >= tiles * (16384 + 1024 + 8192 + 2048 + 512) + Tp * 4 and mx < a
    assert tiles * (16384 + 1024) + Tp * 4 <= sq.sharq_act_bytes(T, K, sq.SHARQ_MODE_MXFP4_PLAIN) < n
    assert sq.sharq_workspace_bytes(16, 256, 256, 1) > 0


def test_views_carve_inside_the_buffer(L):
    base = 1 << 20  # fake, 256-aligned; views never touch memory
    T, K = 300, 768
    n = sq.sharq_act_bytes(T, K, 0)
    a = sq.sharq_act_view(base, T, K, 0)
    ptrs = [a.r_codes, a.r_sf, a.sp_codes, a.meta, a.sp_sf, a.inv_rms, a.s_g, a.gmax_bits]
    assert all(base <= p < base + n for p in ptrs)
    assert len(set(ptrs)) == len(ptrs)
    assert all(p % 16 == 0 for p in ptrs)
    assert (a.T, a.Tp, a.K, a.mode) == (300, 384, 768, 0)
    b = sq.sharq_act_view(base, T, K, 1)
    assert b.sp_codes is None and b.meta is None
    # per-token: the SharQ operands plus Tp per-row scales outside the
    # 256-byte scalar block that holds the sync words
    nt = sq.sharq_act_bytes(T, K, sq.SHARQ_MODE_SHARQ_TOKEN)
    assert nt >= n + 384 * 4
    c = sq.sharq_act_view(base, T, K, sq.SHARQ_MODE_SHARQ_TOKEN)
    assert c.sp_codes and c.meta and c.sp_sf
    assert base <= c.s_g and c.s_g + 384 * 4 <= c.gmax_bits - 16
    assert c.gmax_bits + 240 <= base + nt
    assert c.mode == sq.SHARQ_MODE_SHARQ_TOKEN
    w = sq.sharq_weight_view(base, K, 256, 3)
    assert (w.K, w.D, w.E) == (768, 256, 3)
    assert base <= w.s_w < base + sq.sharq_weight_bytes(K, 256, 3)


def test_argument_errors_before_any_device_work(L):
    with pytest.raises(sq.SharqError) as e:
        sq.sharq_act_view(1 << 20 | 8, 16, 256)           # misaligned
    assert e.value.status == -1
    with pytest.raises(sq.SharqError) as e:
        sq.sharq_act_view(1 << 20, 16, 250)               # K % 256
    assert e.value.status == -2
    a = sq.sharq_act_view(1 << 20, 16, 256)
    w = sq.sharq_weight_view(1 << 24, 512, 256)
    # K mismatch between act and weight
    st = L.sharq_linear(ctypes.byref(a), ctypes.byref(w), 1 << 28, 0, 1 << 29, 256, None)
    assert st == -2
    # bad output dtype
    w2 = sq.sharq_weight_view(1 << 24, 256, 256)
    assert L.sharq_linear(ctypes.byref(a), ctypes.byref(w2), 1 << 28, 9, 1 << 29, 256, None) == -1
    # missing workspace
    assert L.sharq_linear(ctypes.byref(a), ctypes.byref(w2), 1 << 28, 0, None, 0, None) == -6
    # NULL views
    assert L.sharq_prep(1 << 28, None, ctypes.c_float(1e-5), None, None, None) == -1
    assert L.sharq_pack_weight(1 << 28, None, None) == -1
    assert L.sharq_check_status(None, None) == -1
    assert sq.sharq_status_string(-5) == "SHARQ_ERR_TIMEOUT"


def test_layout_round_trip():
    g = np.random.default_rng(0)
    R, K = 256, 512
    codes = g.integers(0, 16, (R, K)).astype(np.uint8)
    assert np.array_equal(_layout.untile_codes(_layout.tile_codes(codes), R, K), codes)
    sp = g.integers(0, 16, (R, K // 2)).astype(np.uint8)
    assert np.array_equal(_layout.untile_sp_codes(_layout.tile_sp_codes(sp), R, K), sp)
    meta = g.integers(0, 16, (R, K // 8)).astype(np.uint8)
    assert np.array_equal(_layout.untile_meta(_layout.tile_meta(meta), R, K), meta)
    for per in (16, 32):
        sf = g.integers(0, 256, (R, K // per)).astype(np.uint8)
        assert np.array_equal(_layout.untile_sf(_layout.tile_sf(sf, per), R, K, per), sf)
    # the first bytes of a codes tile: row 0 is unswizzled, row 1 swaps chunks
    t = _layout.tile_codes(codes[:128, :256])
    assert t[0] == (codes[0, 0] | codes[0, 1] << 4)
    assert t[128 + 16] == (codes[1, 0] | codes[1, 1] << 4)
