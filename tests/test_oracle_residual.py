"""Pins of the oracle's fused residual update h = bf16_rn(f32(x + res)) (CPU).

Pinned against torch's own bfloat16 addition (which adds in float32 and rounds
to nearest even), against the exact float64 sum where the float32 sum is exact,
and by the identities h(x, 0) = x and symmetry.
"""
import numpy as np
import torch

import synthetic
from oracle import sharq


def _bf16(seed, T, K):
    return synthetic.activations(seed, T, K)


def test_matches_torch_bf16_addition():
    x, r = _bf16(1, 16, 512), _bf16(2, 16, 512) * np.float32(8.0)
    h = sharq.residual_add(x, r)
    th = (torch.from_numpy(x).to(torch.bfloat16) + torch.from_numpy(r).to(torch.bfloat16)).float().numpy()
    assert np.array_equal(h, th)


def test_identities():
    x, r = _bf16(3, 8, 256), _bf16(4, 8, 256)
    assert np.array_equal(sharq.residual_add(x, np.zeros_like(x)), x)
    assert np.array_equal(sharq.residual_add(x, r), sharq.residual_add(r, x))
    # values of equal exponent: the float32 sum is exact, h is bf16 of the exact sum
    a = np.array([[1.5, 1.25, -1.75]], np.float32)
    b = np.array([[1.0, 1.0, -1.0]], np.float32)
    assert np.array_equal(sharq.residual_add(a, b), np.array([[2.5, 2.25, -2.75]], np.float32))


def test_equals_exactly_rounded_sum():
    """For two bf16 operands the float32 sum rounded to bf16 is the exactly
    rounded sum (float32 carries more than 2 x 8 + 2 significant bits): checked
    against float64 sums (exact for exponent gaps up to 45) rounded to bf16 by
    torch's float64 -> bfloat16 conversion, over gaps 0..40 and both signs,
    plus hand-made ties (1 + 2^-8 lies halfway between 1 and 1 + 2^-7)."""
    g = np.random.default_rng(5)
    n = 20000
    mant = lambda: (1.0 + g.integers(0, 128, n) / 128.0) * g.choice([-1.0, 1.0], n)
    gap = g.integers(0, 41, n)
    x = (mant() * 2.0 ** g.integers(-20, 20, n)).astype(np.float32)
    r = (mant() * np.ldexp(np.abs(x).astype(np.float64), -gap)).astype(np.float32)
    r = torch.from_numpy(r).to(torch.bfloat16).float().numpy()  # make r a bf16 value
    exact = x.astype(np.float64) + r.astype(np.float64)
    want = torch.from_numpy(exact).to(torch.bfloat16).float().numpy()
    assert np.array_equal(sharq.residual_add(x[None], r[None])[0], want)
    ties = sharq.residual_add(np.array([[1.0, 1.0 + 2 ** -7, -1.0]], np.float32),
                              np.array([[2 ** -8, 2 ** -8, -(2 ** -8)]], np.float32))
    assert np.array_equal(ties, np.array([[1.0, 1.0 + 2 ** -6, -1.0]], np.float32))
