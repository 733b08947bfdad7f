"""Pins of the Table-5 path modes in the oracle (CPU).

xllm-io review, section 5.3 (Table 5) names four ways of splitting the
activation into FP4 operands: Sparse only, Dense+Dense, Sparse+Sparse and
SharQ (sparse backbone + dense residual).  What the mathematics fixes,
independent of any model:
  - rounding to an E2M1 grid that contains 0 (round to nearest, or saturation
    toward the largest grid value) never moves a value farther than 0 does, so
    quantizing a residual can only shrink every element's error:
        |Xn - (B + Q(R))| <= |Xn - B| = |R|   element by element,
    for B the first operand's dequantized values (Dense+Dense against plain
    NVFP4, SharQ and Sparse+Sparse against Sparse only);
  - the residual of an FP4 block is exact in float32 (Sterbenz);
  - Dense+Dense's first level is plain NVFP4 itself;
  - Sparse+Sparse's residual mask keeps exactly 2 of 4 pairs and each chunk's
    largest |R|;
  - the GEMM of SharQ is the Sparse-only GEMM plus the residual GEMM.
The pages' ordering of the modes (Sparse only far worst, Sparse+Sparse near
plain NVFP4, SharQ and Dense+Dense best) is a perplexity result on a real
model; test_reconstruction_error_ordering checks the same ordering on the
synthetic outlier activations as a reported comparison.
"""
import numpy as np

import synthetic
from oracle import sharq
from oracle.formats import e2m1_decode, e4m3_decode


def _x(T=12, K=512, seed=71):
    return synthetic.activations(seed, T, K, n_channels=3, channel_scale=(20.0, 60.0), spike_p=0.01)


def test_dense_dense_first_level_is_plain_nvfp4_and_residual_exact():
    x, g = _x(), synthetic.gamma(72, 512)
    dd = sharq.prep_dense_dense(x, g, 1e-5)
    nv = sharq.prep_nvfp4(x, g, 1e-5)
    assert np.array_equal(dd["b_codes"], nv["codes"]) and np.array_equal(dd["b_sf"], nv["sf"])
    assert np.array_equal(dd["r"].astype(np.float64), dd["xn"].astype(np.float64) - dd["b_t"].astype(np.float64))


def test_elementwise_error_bounds():
    x, g = _x(), synthetic.gamma(73, 512)
    xn, _ = sharq.rmsnorm(x, g, 1e-5)
    xn = xn.astype(np.float64)
    err = {m: np.abs(xn - sharq.approx_activation(x, g, 1e-5, m))
           for m in ("nvfp4", "dense_dense", "sparse_only", "sharq", "sparse_sparse")}
    assert np.all(err["dense_dense"] <= err["nvfp4"])
    assert np.all(err["sharq"] <= err["sparse_only"])
    assert np.all(err["sparse_sparse"] <= err["sparse_only"])
    # and strictly better somewhere (a dropped term would make them equal)
    assert err["dense_dense"].sum() < err["nvfp4"].sum()
    assert err["sharq"].sum() < err["sparse_only"].sum()
    assert err["sparse_sparse"].sum() < err["sparse_only"].sum()


def test_sparse_sparse_residual_mask():
    x = _x(T=6)
    p = sharq.prep_sparse_sparse(x, None, 1e-5)
    keep = p["r_keep"]
    assert np.all(keep.sum(axis=-1) == 2)
    r = np.abs(p["r"].reshape(6, -1, 8))
    kept_el = np.repeat(keep, 2, axis=-1)
    assert np.all((r * kept_el).max(axis=-1) == r.max(axis=-1))
    # where the residual mask drops a pair, nothing of R is represented: the
    # error there is exactly |R|; where it keeps one, the error is below |R|
    dropped = ~np.repeat(keep, 2, axis=-1).reshape(6, -1)
    e = np.abs(p["r"].astype(np.float64) - p["r_sp_t"].astype(np.float64))
    assert np.array_equal(e[dropped], np.abs(p["r"][dropped]).astype(np.float64))
    assert np.all(e[~dropped] <= np.abs(p["r"][~dropped]))
    assert p["r_sp_codes"].shape == (6, 256) and p["r_sp_sf"].shape == (6, 16)


def test_mode_gemms_decompose():
    T, K, D = 5, 512, 128
    x = _x(T=T, K=K)
    wq = sharq.pack_weight(synthetic.weights(74, K, D))
    p = sharq.prep(x, None, 1e-5)
    y = sharq.linear(p, wq)
    w16 = (e2m1_decode(wq["codes"]).reshape(D, K // 16, 16) * e4m3_decode(wq["sf16"])[..., None]).reshape(D, K).T
    y_dense = (sharq.dequant_residual(p) @ w16) * (np.float64(p["s_g"]) * np.float64(wq["s_w"]))
    assert np.allclose(sharq.linear_mode(p, wq, "sparse_only") + y_dense, y, rtol=1e-12, atol=1e-12)
    # Dense+Dense and Sparse+Sparse GEMMs equal X~ W~ of their own operands,
    # up to the float32 rounding of the dequantized X~ (one ulp, 2^-24)
    for mode, prep in (("dense_dense", sharq.prep_dense_dense), ("sparse_sparse", sharq.prep_sparse_sparse)):
        q = prep(x, None, 1e-5)
        a = sharq.approx_activation(x, None, 1e-5, mode)
        ref = a @ wq["w_t"] * np.float64(wq["s_w"])
        got = sharq.linear_mode(q, wq, mode)
        assert np.linalg.norm(got - ref) <= 1e-6 * np.linalg.norm(ref)


def test_reconstruction_error_ordering():
    """Synthetic stand-in for Table 5 (q_proj-shaped outlier activations)."""
    x = synthetic.activations(75, 64, 4096)
    g = synthetic.gamma(76, 4096)
    xn, _ = sharq.rmsnorm(x, g, 1e-5)
    rel = {m: np.linalg.norm(xn - sharq.approx_activation(x, g, 1e-5, m)) / np.linalg.norm(xn)
           for m in ("sparse_only", "nvfp4", "sparse_sparse", "sharq", "dense_dense")}
    assert rel["sparse_only"] > 2 * rel["nvfp4"]
    assert rel["sparse_sparse"] < rel["nvfp4"] < rel["sparse_only"]
    assert rel["sharq"] < 0.5 * rel["nvfp4"]
    assert rel["dense_dense"] < 0.5 * rel["nvfp4"]
