"""Pins of the oracle's MXFP4 variant (CPU).

MXFP4 (OCP Microscaling Formats v1.0): E2M1 elements, one E8M0 scale
X = 2^(floor(log2 amax) - 2) per block.  The xllm-io review, section 5.3, runs
SharQ on MXFP4; on sm_100 the sparse FP4 MMA takes the 4:8 in-pairs pattern and
one E8M0 scale per 64 logical K.  Pinned here without the implementation:
  - the scale rule in closed form (amax / X in [4, 8) for every non-zero block,
    floor(log2) read off the encoding agrees with the logarithm);
  - exact round trip of blocks on the scaled E2M1 grid; saturation;
  - the hand-derived worked example in tests/golden/worked_example_mxfp4.txt;
  - R = (X - X_sp) + (X_sp - X~_sp) exactly, |X - (X~_sp + R~)| <= |R|;
  - the weight's per-32 view repeats the per-64 one (identical values);
  - the GEMM against a pure-Python element loop.
"""
import os

import numpy as np

import synthetic
from oracle import sharq
from oracle.formats import e2m1_decode, e8m0_decode, mx_scale_exponent

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_mxfp4.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if "=" in line:
            k, v = (t.strip() for t in line.split("="))
            out[k] = float(v) if "." in v else int(v, 0)
    return out


def test_scale_rule_closed_form():
    a = np.array([12.0, 0.2001953125, 6.0, 4.0, 7.99, 1.0, 2.0 ** -100, 3.0e38], np.float32)
    e = mx_scale_exponent(a)
    assert np.array_equal(e, np.floor(np.log2(a.astype(np.float64))).astype(np.int64) - 2)
    ratio = a.astype(np.float64) / np.ldexp(1.0, e)
    assert np.all((ratio >= 4) & (ratio < 8))
    assert mx_scale_exponent(np.float32(0.0)) == -127 and mx_scale_exponent(np.float32(1e-40)) == -127
    assert e8m0_decode(127) == 1.0 and e8m0_decode(0) == 2.0 ** -127 and e8m0_decode(254) == 2.0 ** 127


def test_quant_round_trip_and_saturation():
    g = np.random.default_rng(5)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    for k in (-8, 0, 5):
        v = g.choice(grid, (4, 32)) * g.choice([-1.0, 1.0], (4, 32))
        v[:, 0] = 6.0
        v = (v * 2.0 ** k).astype(np.float32)
        c, sb, deq = sharq.mx_quant(v)
        assert np.array_equal(deq.astype(np.float64), v.astype(np.float64))
        assert np.all(sb == k + 127)
    c, sb, deq = sharq.mx_quant(np.array([[7.5] + [0.0] * 31], np.float32))
    assert sb[0] == 127 and c[0, 0] == 7 and deq[0, 0] == 6.0


def test_worked_example():
    G = _golden()
    K = G["K"]
    x = np.full((1, K), G["input_small_bf16"], np.float32)
    x[0, 0] = G["input_outlier"]
    pl = sharq.prep_mxfp4_plain(x, None, 1e-5)
    assert pl["sf"][0, 0] == G["plain_block0_scale_byte"] and pl["sf"][0, 1] == G["plain_block1_scale_byte"]
    assert pl["codes"][0, 0] == G["plain_block0_outlier_code"]
    assert np.all(pl["codes"][0, 1:32] == G["plain_block0_small_code"])
    assert np.all(pl["codes"][0, 32:] == G["plain_block1_code"])
    p = sharq.prep_mxfp4(x, None, 1e-5)
    assert np.all(p["meta"] == G["meta_nibble"])
    assert p["sp_sf"][0, 0] == G["sp_scale_byte"]
    assert p["sp_codes"][0, 0] == G["sp_outlier_code"] and np.all(p["sp_codes"][0, 1:] == G["sp_small_code"])
    assert list(p["r_sf"][0]) == [G["r_scale_byte_block0"], G["r_scale_byte_block1"]]
    assert p["r_codes"][0, 0] == G["r_outlier_code"] and np.all(p["r_codes"][0, 1:] == G["r_small_code"])
    assert np.all(p["r_t"][0, 1:] == np.float32(G["r_small_value"]))


def test_residual_identity_and_bound():
    x = synthetic.activations(61, 8, 512, n_channels=3, channel_scale=(20.0, 60.0), spike_p=0.01)
    g = synthetic.gamma(62, 512)
    p = sharq.prep_mxfp4(x, g, 1e-5)
    xn = p["xn"].astype(np.float64)
    keep_el = np.repeat(p["keep"], 2, axis=-1).reshape(xn.shape)
    assert np.array_equal(p["r"].astype(np.float64),
                          (xn - np.where(keep_el, xn, 0)) + (np.where(keep_el, xn, 0) - p["xsp_t"]))
    approx = p["xsp_t"].astype(np.float64) + p["r_t"].astype(np.float64)
    assert np.all(np.abs(xn - approx) <= np.abs(p["r"]))
    # SharQ beats plain MXFP4 on outlier activations
    pl = sharq.prep_mxfp4_plain(x, g, 1e-5)
    assert np.linalg.norm(xn - approx) < 0.5 * np.linalg.norm(xn - pl["x_t"])


def test_weight_views():
    K, D = 512, 96
    wq = sharq.pack_weight_mx(synthetic.weights(63, K, D))
    assert np.array_equal(wq["sf32"], np.repeat(wq["sf64"], 2, axis=-1))
    d64 = (e2m1_decode(wq["codes"]).reshape(D, K // 64, 64) * e8m0_decode(wq["sf64"])[..., None]).reshape(D, K)
    d32 = (e2m1_decode(wq["codes"]).reshape(D, K // 32, 32) * e8m0_decode(wq["sf32"])[..., None]).reshape(D, K)
    assert np.array_equal(d64, d32) and np.array_equal(d64.T, wq["w_t"])
    assert wq["codes"].shape == (D, K)  # codes are per output column: K != D catches a transpose


def test_linear_against_element_loop():
    T, K, D = 3, 128, 8
    x = synthetic.activations(64, T, K)
    p = sharq.prep_mxfp4(x, None, 1e-5)
    wq = sharq.pack_weight_mx(synthetic.weights(65, K, D))
    y = sharq.linear_mx(p, wq)
    kept = np.repeat(p["keep"], 2, axis=-1).reshape(T, K)
    for t in range(T):
        idx = 0
        a_sp = [0.0] * K
        for k in range(K):
            if kept[t, k]:
                a_sp[k] = float(e2m1_decode(p["sp_codes"][t, idx])) * 2.0 ** (int(p["sp_sf"][t, idx // 32]) - 127)
                idx += 1
        for d in range(D):
            acc = 0.0
            for k in range(K):
                wv = float(e2m1_decode(wq["codes"][d, k])) * 2.0 ** (int(wq["sf64"][d, k // 64]) - 127)
                rv = float(e2m1_decode(p["r_codes"][t, k])) * 2.0 ** (int(p["r_sf"][t, k // 32]) - 127)
                acc += (a_sp[k] + rv) * wv
            assert abs(acc - y[t, d]) <= 1e-12 * max(1.0, abs(acc))
