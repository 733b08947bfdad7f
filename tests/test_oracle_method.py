"""Pins for the oracle's method steps (CPU only).

Each test pins one step to something other than the oracle itself: brute
force, closed forms, library routines, the identities and bound of the xllm-io
review's section 3.6, and the kasblo.com explainer's worked example.
"""
import itertools
import os

import numpy as np
import pytest
import torch

import synthetic
from oracle import sharq
from oracle.formats import e2m1_decode, e4m3_decode

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if "=" in line:
                k, v = (s.strip() for s in line.split("=", 1))
                out[k] = float(int(v, 16)) if v.startswith("0x") else float(v)
    return out

# ------------------------------------------------------------------ mask ---


def test_pair_mask_brute_force_all_score_tuples():
    """All 81 score 4-tuples in {0,1,2}^4 against a sort-based rule."""
    tuples = list(itertools.product([0.0, 1.0, 2.0], repeat=4))
    xn = np.zeros((len(tuples), 8), dtype=np.float32)
    for i, t in enumerate(tuples):
        for p, s in enumerate(t):
            # put the score in the second slot of the pair with a negative sign
            # to check that magnitudes are compared
            xn[i, 2 * p + 1] = -s
            xn[i, 2 * p] = s / 2
    keep, meta = sharq.pair_mask(xn)
    for i, t in enumerate(tuples):
        order = sorted(range(4), key=lambda p: (-t[p], p))
        want = sorted(order[:2])
        got = [p for p in range(4) if keep[i, 0, p]]
        assert got == want, (t, got, want)
        assert meta[i, 0] == want[0] | (want[1] << 2)


def test_pair_mask_keeps_exactly_two_pairs_and_chunk_max():
    x = synthetic.activations(11, 64, 512)
    keep, meta = sharq.pair_mask(x)
    assert np.all(keep.sum(-1) == 2)                  # 4:8 in pairs
    lo, hi = meta & 3, meta >> 2
    assert np.all(lo < hi)
    a = np.abs(x.reshape(64, 64, 8))
    top = np.argmax(a, axis=-1) // 2
    assert np.all(np.take_along_axis(keep, top[..., None], -1))

# --------------------------------------------------------------- rmsnorm ---


def test_rmsnorm_closed_form_constant_row():
    K = 256
    x = np.full((3, K), 2.0, dtype=np.float32)
    x[1] = -0.5
    x[2] = 0.0
    g = np.full(K, 1.0, dtype=np.float32)
    xn, inv = sharq.rmsnorm(x[:2], g, 0.0)
    assert inv[0] == np.float32(0.5) and inv[1] == np.float32(2.0)
    assert np.all(xn[0] == 1.0) and np.all(xn[1] == -1.0)
    xn, inv = sharq.rmsnorm(x[2:], g, 1e-6)
    assert np.all(xn == 0.0)


def test_rmsnorm_matches_torch_within_one_bf16_ulp():
    x = synthetic.activations(12, 32, 1024)
    g = synthetic.gamma(13, 1024)
    xn, _ = sharq.rmsnorm(x, g, 1e-5)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (1024,),
                                       torch.from_numpy(g).double(), eps=1e-5)
    ref = ref.numpy()
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(xn - ref) <= ulp)


def test_rmsnorm_off_is_identity():
    x = synthetic.activations(14, 4, 256)
    xn, inv = sharq.rmsnorm(x, None, 1e-5)
    assert inv is None and np.array_equal(xn, x)

# ------------------------------------------------------------------- PTS ---


def test_pts_closed_form():
    x = np.zeros((2, 32), dtype=np.float32)
    s, g = sharq.pts_scale(x)
    assert s == 1.0 and g == 0.0
    x[1, 7] = -2688.0
    s, g = sharq.pts_scale(x)
    assert g == 2688.0 and s == 1.0
    x[1, 7] = 12.0
    s, _ = sharq.pts_scale(x)
    assert s == np.float32(np.float32(12.0) / np.float32(2688.0))

# ------------------------------------------------------------- quantizer ---


def test_nvfp4_round_trip_exact_on_grid():
    """Values exactly on grid*S reconstruct exactly when S is representable."""
    s = np.float32(0.25)
    vals = np.array([6, -4, 3, 0.5, -1.5, 2, 0, 1, -6, 4, 1.5, -3, 0.5, -0.5, 2, 1],
                    dtype=np.float32)
    v = (vals * np.float32(3.0) * s)[None, :]   # block scale 3 (exact E4M3)
    codes, sb, deq = sharq.nvfp4_quant(v, s)
    assert e4m3_decode(sb)[0] == 3.0
    assert np.array_equal(e2m1_decode(codes[0]), vals.astype(np.float64))
    assert np.array_equal(deq, v)


def test_nvfp4_zero_block_and_error_bound():
    codes, sb, deq = sharq.nvfp4_quant(np.zeros((1, 16), np.float32), np.float32(1.0))
    assert np.all(codes == 0) and sb[0] == 0 and np.all(deq == 0)
    g = np.random.default_rng(5)
    v = (g.standard_normal((4000, 16)) * np.exp(g.uniform(-3, 3, (4000, 1)))).astype(np.float32)
    s = np.float32(np.max(np.abs(v)) / 2688.0)
    codes, sb, deq = sharq.nvfp4_quant(v, s)
    S = e4m3_decode(sb) * np.float64(s)
    # largest grid gap is 2 (between 4 and 6), so rounding error <= S; the scale
    # rounding (3 mantissa bits) can push |v|/S above 6 by at most 1/16 -> +6S/16
    err = np.abs(v - deq)
    assert np.all(err <= S[:, None] * (1.0 + 6.0 / 16.0) + 1e-6 * np.abs(v))

# ------------------------------------------------ residual and analysis ---


def _small_case(seed=21, T=8, K=256):
    x = synthetic.activations(seed, T, K, n_channels=4, channel_scale=(30.0, 30.0),
                              spike_p=0.01)
    return x


def test_prep_structure_and_residual_identity():
    """R = (X - X_sp) + (X_sp - X~_sp) exactly (xllm-io review, section 3.3),
    R = Xn where the mask drops a value (kasblo.com explainer: sparsity routes
    values to the residual instead of dropping them)."""
    x = _small_case()
    g = synthetic.gamma(22, 256)
    p = sharq.prep(x, g, 1e-5)
    T, K = x.shape
    keep_el = np.repeat(p["keep"], 2, -1).reshape(T, K)
    assert np.array_equal(p["xsp"], np.where(keep_el, p["xn"], 0))
    assert np.array_equal(p["r"][~keep_el], p["xn"][~keep_el])
    x64, xsp64, xt64 = (p[k].astype(np.float64) for k in ("xn", "xsp", "xsp_t"))
    assert np.array_equal(p["r"].astype(np.float64), (x64 - xsp64) + (xsp64 - xt64))
    # the sparse-path block amax equals the full 32-element block amax
    spa = np.max(np.abs(p["sp_vals"].reshape(T, K // 32, 16)), -1)
    fulla = np.max(np.abs(p["xn"].reshape(T, K // 32, 32)), -1)
    assert np.array_equal(spa, fulla)


def test_error_merge_identity_and_output_bound():
    """X - (X~_sp + R~) = R - R~ and ||X W - (X~_sp + R~) W||_F <= ||R - R~||_F ||W||_2
    (xllm-io review, section 3.6), in float64 with W = dequantized weight."""
    x = _small_case(31, 16, 256)
    w = synthetic.weights(32, 256, 96)
    p = sharq.prep(x, None)
    wq = sharq.pack_weight(w)
    s_g = np.float64(p["s_g"])
    xsp_t = sharq.dequant_sparse(p) * s_g
    r = p["xn"].astype(np.float64) - xsp_t
    r_t = sharq.dequant_residual(p) * s_g
    lhs = p["xn"].astype(np.float64) - (xsp_t + r_t)
    assert np.allclose(lhs, r - r_t, rtol=0, atol=1e-12)
    wbar = wq["w_t"] * np.float64(wq["s_w"])
    err = np.linalg.norm(p["xn"] @ wbar - (xsp_t + r_t) @ wbar)
    bound = np.linalg.norm(r - r_t) * np.linalg.norm(wbar, 2)
    assert err <= bound * (1 + 1e-12)
    # and the dual-path GEMM equals (X~_sp + R~) W~ (section 3.4)
    y = sharq.linear(p, wq)
    assert np.allclose(y, (xsp_t + r_t) @ wbar, rtol=1e-12, atol=1e-12)


def test_worked_example_outlier_isolation():
    gd = _golden("worked_example.txt")
    K = int(gd["K"])
    x = np.full((1, K), gd["input_small_bf16"], dtype=np.float32)
    x[0, 0] = gd["input_outlier"]
    assert gd["nvfp4_bits_per_16"] == 16 * 4 + 8
    assert gd["nvfp4_bits_per_value"] == gd["nvfp4_bits_per_16"] / 16
    plain = sharq.prep_nvfp4(x, None)
    assert plain["sf"][0, 0] == gd["plain_block0_scale_byte"]
    assert plain["codes"][0, 0] == gd["plain_block0_outlier_code"]
    assert np.all(plain["codes"][0, 1:16] == gd["plain_block0_small_code"])
    p = sharq.prep(x, None)
    assert np.all(p["meta"] == gd["meta_nibble"])
    assert p["sp_sf"][0, 0] == gd["sp_scale_byte"]
    assert p["sp_codes"][0, 0] == gd["sp_outlier_code"]
    assert np.all(p["sp_codes"][0, 2:] == gd["sp_small_code"])
    assert p["r_sf"][0, 0] == gd["r_scale_byte"]
    assert np.all(p["r_codes"][0, 1:] == gd["r_small_code"])
    ratio = e4m3_decode(p["sp_sf"][0, 0]) / e4m3_decode(p["r_sf"][0, 0])
    assert abs(ratio - gd["scale_shrink"]) < 1e-5
    # SharQ keeps the small values that plain NVFP4 erased in the outlier's block
    plain_err = np.abs(plain["x_t"][0, 1:16] - x[0, 1:16]).max()
    sharq_err = np.abs((p["xsp_t"] + p["r_t"])[0, 1:16] - x[0, 1:16]).max()
    assert plain_err == pytest.approx(gd["input_small_bf16"])
    assert sharq_err < 0.01 * gd["input_small_bf16"]

# ----------------------------------------------------------------- GEMM ----


def _loop_linear(p, wq):
    """Pure-python restatement of Y from the logical codes, one element at a
    time: decompress each activation position through the mask, decode both
    operands, multiply-accumulate."""
    T, K = p["xn"].shape
    D = wq["codes"].shape[0]
    e2 = [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]

    def e4(b):
        e, m = (b >> 3) & 15, b & 7
        return (m / 8) * 2 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    y = np.zeros((T, D))
    for t in range(T):
        a = [0.0] * K
        for k in range(K):
            c, pr = k // 8, (k % 8) // 2
            m = int(p["meta"][t, c])
            kept = [m & 3, m >> 2]
            if pr in kept:
                slot = kept.index(pr)
                j = c * 4 + slot * 2 + k % 2
                a[k] += e2[p["sp_codes"][t, j]] * e4(int(p["sp_sf"][t, j // 16]))
            a[k] += e2[p["r_codes"][t, k]] * e4(int(p["r_sf"][t, k // 16]))
        for d in range(D):
            acc = 0.0
            for k in range(K):
                w = e2[wq["codes"][d, k]] * e4(int(wq["sf16"][d, k // 16]))
                acc += a[k] * w
            y[t, d] = acc * float(p["s_g"]) * float(wq["s_w"])
    return y


def test_linear_matches_pure_python_loop():
    x = _small_case(41, 3, 64)
    w = synthetic.weights(42, 64, 5)
    p = sharq.prep(x, synthetic.gamma(43, 64), 1e-6)
    wq = sharq.pack_weight(w)
    y = sharq.linear(p, wq)
    assert np.allclose(y, _loop_linear(p, wq), rtol=1e-12, atol=1e-12)
    # and close to the unquantized product (sanity of scale placement)
    y_ref = p["xn"].astype(np.float64) @ w.astype(np.float64)
    assert np.linalg.norm(y - y_ref) < 0.2 * np.linalg.norm(y_ref)


def test_pack_weight_views_and_bound():
    w = synthetic.weights(51, 128, 48)          # K != D catches a transpose
    wq = sharq.pack_weight(w)
    assert wq["codes"].shape == (48, 128)
    assert np.array_equal(wq["sf16"], np.repeat(wq["sf32"], 2, axis=1))
    S = e4m3_decode(wq["sf32"]) * np.float64(wq["s_w"])       # [D, K/32]
    err = np.abs(wq["w_t"] * np.float64(wq["s_w"]) - w)       # [K, D]
    bound = np.repeat(S, 32, axis=1).T * (1.0 + 6.0 / 16.0)
    assert np.all(err <= bound + 1e-9)
    assert wq["s_w"] == np.float32(np.float32(np.max(np.abs(w))) / np.float32(2688))


def test_sharq_beats_plain_nvfp4_on_outlier_data():
    """The decomposition's purpose (xllm-io review, section 3.6): with channel
    outliers the sparse+dense pair reconstructs X better than plain NVFP4."""
    x = synthetic.activations(61, 64, 1024, channel_frac=0.005, channel_scale=(20, 60))
    p = sharq.prep(x, None)
    plain = sharq.prep_nvfp4(x, None)
    e_sharq = np.linalg.norm(p["xsp_t"].astype(np.float64) + p["r_t"] - x)
    e_plain = np.linalg.norm(plain["x_t"].astype(np.float64) - x)
    assert e_sharq < 0.5 * e_plain


def test_grouped_equals_per_expert():
    x = _small_case(71, 40, 256)
    p = sharq.prep(x, None)
    wqs = [sharq.pack_weight(synthetic.weights(72 + e, 256, 32)) for e in range(3)]
    offs = np.array([0, 13, 13, 40])
    y = sharq.linear_grouped(p, wqs, offs)
    for e in range(3):
        lo, hi = offs[e], offs[e + 1]
        if hi > lo:
            sub = {k: (v[lo:hi] if isinstance(v, np.ndarray) and v.ndim and v.shape[0] == 40 else v)
                   for k, v in p.items()}
            assert np.array_equal(y[lo:hi], sharq.linear(sub, wqs[e]))
