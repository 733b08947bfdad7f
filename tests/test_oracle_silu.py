"""Pins of the oracle's SwiGLU epilogue h = bf16(silu_bf16(gate) * up) (CPU).

The down projection of a Llama-style MLP takes SiLU(gate) * up; the kasblo.com
explainer (section 4, on fusing the preparation) counts the epilogues before
the preparation among what the prep kernel takes in.  silu_bf16 is read as the
correctly rounded bfloat16 of silu(g) = g / (1 + e^-g).  What pins it:
  - every one of the 65536 bf16 inputs against the correctly rounded value
    from 60-digit decimal arithmetic (nearest bf16, with the neighbours
    compared exactly): an exhaustive check, so no input is left out;
  - the special values (signed zeros, infinities, NaN, the saturating tails);
  - the product against torch's own bf16 F.silu(gate) * up, which agrees
    wherever torch's SiLU is itself correctly rounded;
  - multiplying by 1 returns the SiLU itself.
"""
from decimal import Decimal, localcontext

import numpy as np
import torch

import synthetic
from oracle import sharq


def _all_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    return bits, v


PREC = 120  # digits: silu(g) - g/2 ~ g^2/4 must survive next to g/2 for g ~ 2^-133


def _exact_silu(gv):
    g = Decimal(float(gv))
    if g >= 0:
        return g / (1 + (-g).exp())
    e = g.exp()
    return g * e / (1 + e)


def test_exhaustive_correct_rounding():
    bits, v = _all_bf16()
    fin = np.isfinite(v)
    got = sharq.silu_bf16(v)
    gbits = (got.view(np.uint32) >> 16).astype(np.int64)
    assert np.all((got.view(np.uint32) & 0xFFFF) == 0)  # bf16 values
    bad = []
    with localcontext() as c:
        c.prec = PREC
        _check_all(v, fin, got, gbits, bits, bad)
    assert not bad, f"{len(bad)} inputs not correctly rounded, first {bad[:5]}"


def _check_all(v, fin, got, gbits, bits, bad):
    for i in np.nonzero(fin)[0]:
        S = _exact_silu(v[i])
        neg = bool(np.signbit(v[i]))
        assert bool(np.signbit(got[i])) == neg, (hex(bits[i]), got[i])
        mag = gbits[i] & 0x7FFF
        cand = Decimal(float(np.uint32(mag << 16).view(np.float32)))
        up = Decimal(float(np.uint32((mag + 1) << 16).view(np.float32))) if mag < 0x7F7F else None
        down = Decimal(float(np.uint32((mag - 1) << 16).view(np.float32))) if mag > 0 else None
        a = abs(S)
        ok = (up is None or abs(a - cand) < abs(a - up)) and (down is None or abs(a - cand) < abs(a - down))
        if not ok:
            bad.append(hex(bits[i]))


def test_special_values():
    g = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 3.0e38, -3.0e38, 2.0 ** 20, -(2.0 ** 20)], np.float32)
    s = sharq.silu_bf16(g)
    assert s[0] == 0 and not np.signbit(s[0]) and s[1] == 0 and np.signbit(s[1])
    assert s[2] == np.inf and s[3] == 0 and np.signbit(s[3]) and np.isnan(s[4])
    assert s[5] == np.float32(sharq.bf16_round(np.float32(3.0e38))) and s[6] == 0 and np.signbit(s[6])
    assert s[7] == np.float32(2.0 ** 20) and s[8] == 0 and np.signbit(s[8])
    # the smallest subnormal: silu(g) = g/2 + (g/2) tanh(g/2) lies just above the
    # midpoint g/2 between 0 and g, so it rounds up to g; for -g, toward zero
    tiny = np.float32(2.0 ** -133)
    assert sharq.silu_bf16(np.array([tiny]))[0] == tiny
    t = sharq.silu_bf16(np.array([-tiny]))[0]
    assert t == 0 and np.signbit(t)


def test_product_matches_torch_bf16():
    g = synthetic.activations(31, 64, 512) * np.float32(0.25)
    u = synthetic.activations(32, 64, 512)
    h = sharq.silu_mul(g, u)
    tg, tu = torch.from_numpy(g).to(torch.bfloat16), torch.from_numpy(u).to(torch.bfloat16)
    th = (torch.nn.functional.silu(tg) * tu).float().numpy()
    ts = torch.nn.functional.silu(tg).float().numpy()
    own = sharq.silu_bf16(g)
    differ = h != th
    # where they differ, torch's bf16 SiLU is not the correctly rounded one
    assert np.all(ts[differ] != own[differ])
    assert differ.mean() < 1e-3
    assert np.array_equal(h[~differ], th[~differ])


def test_times_one_is_silu():
    g = synthetic.activations(33, 8, 256)
    assert np.array_equal(sharq.silu_mul(g, np.ones_like(g)), sharq.silu_bf16(g))


def test_bf16_round_f64_matches_torch_conversion():
    """One rounding from float64 to bf16 (not through float32): checked
    against torch's float64 -> bfloat16 conversion on values spread over the
    normal and subnormal range, including exact halfway cases."""
    g = np.random.default_rng(9)
    x = g.standard_normal(20000) * np.exp2(g.integers(-140, 120, 20000).astype(np.float64))
    halfway = (np.arange(1, 200, dtype=np.float64) * 2 + 1) * 2.0 ** -9  # odd multiples of half a bf16 ulp at 1
    x = np.concatenate([x, halfway, -halfway, [0.0, -0.0, 2.0 ** -134, 3 * 2.0 ** -134]])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = sharq.bf16_round_f64(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
