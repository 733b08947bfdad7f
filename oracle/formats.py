"""Number formats used by NVFP4, written from their definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

NVFP4 (kasblo.com explainer, section "FP4 block scale is dominated by outliers"):
16 E2M1 values share one FP8-E4M3 scale, 16*4 + 8 = 72 bits per 16 values,
4.5 bits per value.  The xllm-io review, section 3.1, adds the second-level
FP32 global scale.

E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no Inf/NaN.
  magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
E4M3 (the "FN" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
  bits, no Inf, S.1111.111 is NaN, largest finite 448, smallest subnormal 2^-9.

Rounding: round to nearest, ties to the even code (the code whose mantissa LSB
is 0), and saturate magnitudes above the largest finite value to it (the
"satfinite" behaviour).  The sign of an E2M1 result is the sign of the input,
so a negative input that rounds to zero gives code 0b1000.
"""
import numpy as np

# ---------------------------------------------------------------- E2M1 -----


def e2m1_decode(code):
    """Value of each 4-bit E2M1 code (array of ints 0..15) as float64."""
    code = np.asarray(code, dtype=np.int64)
    sign = np.where(code & 8, -1.0, 1.0)
    e = (code >> 1) & 3
    m = code & 1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e - 1.0))
    return sign * mag


E2M1_GRID = e2m1_decode(np.arange(8))  # 0, .5, 1, 1.5, 2, 3, 4, 6


def e2m1_encode(x):
    """Round float32 values to E2M1 codes (RNE, ties to even code, satfinite).

    Brute force over the 8 magnitudes: pick the nearest; on an exact tie pick
    the even code.  Inputs are exact binary fractions, so float64 distances
    are exact.
    """
    x = np.asarray(x, dtype=np.float32)
    mag = np.abs(x.astype(np.float64))
    dist = np.abs(mag[..., None] - E2M1_GRID)            # [..., 8]
    best = np.argmin(dist, axis=-1)                      # first minimum
    dmin = np.take_along_axis(dist, best[..., None], -1)[..., 0]
    # an exact tie can only be with the next code up; prefer the even one
    nxt = np.minimum(best + 1, 7)
    dn = np.take_along_axis(dist, nxt[..., None], -1)[..., 0]
    tie = (nxt != best) & (dn == dmin) & (best % 2 == 1)
    best = np.where(tie, nxt, best)
    best = np.where(mag > 6.0, 7, best)                  # satfinite
    sign = np.signbit(x).astype(np.int64) << 3
    return (best + sign).astype(np.uint8)

# ---------------------------------------------------------------- E4M3 -----


def e4m3_decode(b):
    """Value of each E4M3 byte as float64 (NaN for S.1111.111)."""
    b = np.asarray(b, dtype=np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 15
    m = b & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((b & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_decode(np.arange(0x7F))  # bytes 0x00..0x7E, increasing


def e4m3_encode_nonneg(x):
    """Round non-negative float32 values to E4M3 bytes (RNE, satfinite)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.any(x < 0) or np.any(np.isnan(x)):
        raise ValueError("e4m3_encode_nonneg takes non-negative finite values")
    hi = np.searchsorted(_E4M3_POS, x, side="left")      # first value >= x
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    dhi = np.abs(_E4M3_POS[hi] - x)
    dlo = np.abs(x - _E4M3_POS[lo])
    pick = np.where(dlo < dhi, lo, hi)
    tie = (dlo == dhi) & (lo != hi)
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    pick = np.where(x >= 448.0, 0x7E, pick)              # satfinite
    return pick.astype(np.uint8)

# ---------------------------------------------------------------- bf16 -----


# ---------------------------------------------------------------- E8M0 -----
# The MX scale type (OCP Microscaling Formats specification v1.0, "E8M0"):
# 8 exponent bits, bias 127, no sign, no mantissa; 0xFF is NaN.  Byte e is
# 2^(e - 127).  MXFP4 (the same specification) is 32 E2M1 elements sharing
# one E8M0 scale X = 2^(floor(log2(amax)) - emax_elem), emax_elem = 2 for
# E2M1 (largest normal 6 = 1.5 * 2^2); the elements are x / X rounded to
# E2M1 (round to nearest even, saturating).


def e8m0_decode(b):
    """Value of each E8M0 byte (array of ints 0..254) as float64."""
    b = np.asarray(b, dtype=np.int64)
    return np.ldexp(1.0, b - 127)


def mx_scale_exponent(amax):
    """Shared exponent of an MX block from its float32 amax: floor(log2(amax))
    - 2, clamped to the E8M0 range [-127, 127]; -127 for an all-zero block.
    floor(log2) is read off the float32 encoding exactly (no logarithm)."""
    a = np.asarray(amax, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.int64)
    e_field = (bits >> 23) & 0xFF
    mant = bits & 0x7FFFFF
    # normal: e_field - 127; subnormal: position of the highest mantissa bit
    sub = np.where(mant > 0, np.floor(np.log2(np.maximum(mant, 1))).astype(np.int64) - 149, -1000)
    fl = np.where(e_field > 0, e_field - 127, sub)
    e = np.where(a > 0, fl - 2, -127)
    return np.clip(e, -127, 127)


def bf16_round(x):
    """Round float32 to the nearest bfloat16 (ties to even); returns float32.

    bfloat16 is the top 16 bits of a float32.  Finite inputs only.
    """
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def f32(x):
    """Round to float32 (one IEEE rounding from float64)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)
