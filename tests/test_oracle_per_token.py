"""Pins of the oracle's per-token global-scale reading (CPU).

The pages never expand "PTS" (xllm-io review, sections 3.1 and 3.5); the
per-token reading gives every row its own s_t = max|Xn[t]| / (6*448).  What
that reading fixes, and what a per-tensor scale would break:
  - rows are prepared independently: any subset of rows prepares exactly as
    the same rows of the whole tensor, even when the subset leaves out the
    row that holds the tensor's maximum;
  - scaling one row (no RMSNorm) by a power of two scales that row's s_t by
    the same power and leaves every code, scale byte and mask unchanged -- in
    every row, the scaled one included;
  - a one-row tensor is prepared exactly as by the per-tensor prep;
  - Y row t carries the factor s_t: scaling row t of X by 2^k scales row t of
    Y by 2^k and no other row.
"""
import numpy as np

import synthetic
from oracle import sharq

FIELDS = ("meta", "sp_codes", "sp_sf", "r_codes", "r_sf")


def _x(T=9, K=256, seed=41):
    x = synthetic.activations(seed, T, K, n_channels=4, channel_scale=(20.0, 60.0), spike_p=0.01)
    if T > 3:
        x[3] *= 64.0  # one row far above the others (a power of two keeps bf16 values)
    return x.astype(np.float32)


def test_single_row_equals_per_tensor():
    x = _x(T=1)
    g = synthetic.gamma(3, x.shape[1])
    a = sharq.prep_per_token(x, g, 1e-5)
    b = sharq.prep(x, g, 1e-5)
    assert a["s_g"].shape == (1,) and a["s_g"][0] == b["s_g"]
    for f in FIELDS:
        assert np.array_equal(a[f], b[f]), f


def test_subsets_of_rows_prepare_independently():
    x = _x()
    g = synthetic.gamma(4, x.shape[1])
    whole = sharq.prep_per_token(x, g, 1e-6)
    rows = [0, 2, 5, 8]  # leaves out row 3, the tensor's maximum
    part = sharq.prep_per_token(x[rows], g, 1e-6)
    assert np.array_equal(part["s_g"], whole["s_g"][rows])
    for f in FIELDS:
        assert np.array_equal(part[f], whole[f][rows]), f
    # the per-tensor reading does not have this property on this input
    pt_whole, pt_part = sharq.prep(x, g, 1e-6), sharq.prep(x[rows], g, 1e-6)
    assert not np.array_equal(pt_part["r_sf"], pt_whole["r_sf"][rows])


def test_power_of_two_row_scaling():
    x = _x()
    k = 3
    y = x.copy()
    y[5] *= np.float32(2.0 ** k)
    a = sharq.prep_per_token(x, None, 1e-5)
    b = sharq.prep_per_token(y, None, 1e-5)
    assert b["s_g"][5] == np.float32(a["s_g"][5] * 2.0 ** k)
    others = [t for t in range(x.shape[0]) if t != 5]
    assert np.array_equal(b["s_g"][others], a["s_g"][others])
    for f in FIELDS:
        assert np.array_equal(a[f], b[f]), f


def test_all_zero_row_gets_unit_scale():
    x = _x(T=3)
    x[1] = 0.0
    p = sharq.prep_per_token(x, None, 1e-5)
    assert p["s_g"][1] == np.float32(1.0)
    assert not p["sp_codes"][1].any() and not p["r_codes"][1].any()


def test_linear_row_scale():
    T, K, D = 6, 256, 128
    x = _x(T=T, K=K)
    wq = sharq.pack_weight(synthetic.weights(5, K, D))
    y0 = sharq.linear(sharq.prep_per_token(x, None, 1e-5), wq)
    x2 = x.copy()
    x2[2] *= np.float32(8.0)
    y1 = sharq.linear(sharq.prep_per_token(x2, None, 1e-5), wq)
    assert np.array_equal(y1[2], y0[2] * 8.0)
    rest = [t for t in range(T) if t != 2]
    assert np.array_equal(y1[rest], y0[rest])
    # and every row equals the per-tensor product of that row alone
    for t in range(T):
        yt = sharq.linear(sharq.prep(x[t:t + 1], None, 1e-5), wq)
        assert np.array_equal(yt[0], y0[t])
