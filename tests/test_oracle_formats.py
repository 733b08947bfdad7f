"""Pins for the oracle's number formats (CPU only).

The E2M1 / E4M3 / bf16 routines are checked against the format definitions
(tables typed from the definitions), against hand-listed rounding ties, and
against two independent library implementations (ml_dtypes, torch).
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle.formats import (bf16_round, e2m1_decode, e2m1_encode, e4m3_decode,
                            e4m3_encode_nonneg)


def test_e2m1_table_matches_definition():
    # sign | exponent(2) | mantissa(1); grid {0, .5, 1, 1.5, 2, 3, 4, 6}
    expect = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    expect = expect + [-v for v in expect]
    got = e2m1_decode(np.arange(16))
    assert np.array_equal(got, np.array(expect))
    assert np.signbit(got[8])


@pytest.mark.parametrize("x,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
    (0.2500001, 1), (0.7499999, 1), (5.0000005, 7), (6.0, 7), (7.0, 7), (1e30, 7),
    (-0.25, 8), (-0.1, 8), (-0.0, 8), (0.0, 0), (-5.0, 14), (-6.5, 15),
])
def test_e2m1_ties_and_saturation(x, code):
    assert int(e2m1_encode(np.float32(x))) == code


def test_e2m1_matches_ml_dtypes():
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    mids = (grid[1:] + grid[:-1]) / 2
    pts = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, 10),
                          [6.5, 7, 100, 1e-8]]).astype(np.float32)
    rnd = np.random.default_rng(1).uniform(-8, 8, 20000).astype(np.float32)
    x = np.concatenate([pts, -pts, rnd]).astype(np.float32)
    ours = e2m1_encode(x)
    lib = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, lib)


def test_e4m3_decode_all_bytes():
    b = np.arange(256)
    ours = e4m3_decode(b)
    lib = b.astype(np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0
    assert ours[0x08] == 2.0 ** -6 and ours[0x4F] == 7.5


def test_e4m3_encode_matches_torch_and_saturates():
    vals = e4m3_decode(np.arange(0x7F))
    mids = (vals[1:] + vals[:-1]) / 2
    rnd = np.random.default_rng(2).uniform(0, 448, 50000)
    tiny = np.random.default_rng(3).uniform(0, 2 ** -5, 5000)
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rnd, tiny]).astype(np.float32)
    x = x[x <= 448]
    ours = e4m3_encode_nonneg(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    big = np.array([448.0, 449, 464, 480, 1e6], dtype=np.float32)
    assert np.all(e4m3_encode_nonneg(big) == 0x7E)


def test_bf16_round_matches_torch():
    g = np.random.default_rng(4)
    x = np.concatenate([g.standard_normal(100000) * 10.0 ** g.integers(-20, 20, 100000),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8]]).astype(np.float32)
    ours = bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
