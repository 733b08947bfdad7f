"""End-to-end parity: sharq_prep + sharq_linear vs the oracle (GPU).

Y is compared with the oracle's float64 product of the same quantized
operands (xllm-io review, section 3.4).  Tolerances:
  - float32 output: relative Frobenius error <= 1e-3 (the contract), and in
    practice ~1e-6 (float32 accumulation only);
  - bf16 output: the rounding to bf16 alone costs up to 2^-8 relative per
    element (bf16 keeps 8 significant bits), so each element must be within
    2^-8 |y| + 1e-4 max|y| of the float64 reference and the relative
    Frobenius error within 1e-3 + 2^-8.
"""
import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
import synthetic
from oracle import sharq as O
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

F32_TOL = 1e-3
BF16_FRO_TOL = 1e-3 + 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def _run(x, gamma, eps, w, mode=sq.SHARQ_MODE_SHARQ, out_dtype=torch.float32):
    T, K = x.shape
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    act = sq.PreparedAct(T, K, mode)
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma) if gamma is not None else None, eps)
    ws = sq.Workspace(T, K, w.shape[1])
    y = sq.linear(act, pw, out_dtype=out_dtype, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    return y.float().cpu().numpy()


CASES = [
    ("single_linear_T16_K256_D256", 16, 256, 256, dict(n_channels=4, channel_scale=(30.0, 30.0), spike_p=0.01), "one"),
    ("q_proj_T1", 1, 4096, 4096, dict(), "uniform"),
    ("q_proj_T16", 16, 4096, 4096, dict(), "uniform"),
    ("ragged_T200_K768_D384", 200, 768, 384, dict(), "uniform"),
    ("down_T130_K1536_D512", 130, 1536, 512, dict(base="student_t"), None),
]


@pytest.mark.parametrize("name,T,K,D,kw,gam", CASES, ids=[c[0] for c in CASES])
def test_linear_matches_oracle(name, T, K, D, kw, gam):
    x = synthetic.activations(200 + T, T, K, **kw)
    gamma = None if gam is None else (synthetic.gamma(3, K, 1.0, 1.0) if gam == "one" else synthetic.gamma(4, K))
    w = synthetic.weights(300 + D, K, D)
    p = O.prep(x, gamma, 1e-5)
    q = O.pack_weight(w)
    ref = O.linear(p, q)
    y32 = _run(x, gamma, 1e-5, w)
    e32 = H.rel_fro(y32, ref)
    assert e32 <= F32_TOL, e32
    assert e32 < 1e-5, f"float32 path should only carry accumulation error, got {e32}"
    yb = _run(x, gamma, 1e-5, w, out_dtype=torch.bfloat16)
    assert H.rel_fro(yb, ref) <= BF16_FRO_TOL
    assert np.all(np.abs(yb - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max())


def test_nvfp4_comparator_matches_oracle():
    T, K, D = 64, 1024, 256
    x = synthetic.activations(7, T, K)
    gamma = synthetic.gamma(8, K)
    w = synthetic.weights(9, K, D)
    ref = O.linear_nvfp4(O.prep_nvfp4(x, gamma, 1e-5), O.pack_weight(w))
    y = _run(x, gamma, 1e-5, w, mode=sq.SHARQ_MODE_NVFP4)
    assert H.rel_fro(y, ref) < 1e-5


def test_sharq_error_below_nvfp4_on_outliers():
    """The point of the method (xllm-io review, section 3.6), measured on the
    GPU outputs: with the same FP4 weights W~, the activation-side error of
    SharQ, ||Xn W~ - Y||, is well below plain NVFP4's on outlier activations.
    (Against the unquantized X W both carry the same weight error, which
    hides the difference.)"""
    T, K, D = 128, 2048, 512
    x = synthetic.activations(10, T, K, channel_frac=0.005, channel_scale=(20, 60))
    w = synthetic.weights(11, K, D)
    q = O.pack_weight(w)
    xw = x.astype(np.float64) @ (q["w_t"] * np.float64(q["s_w"]))
    ys = _run(x, None, 1e-5, w)
    yn = _run(x, None, 1e-5, w, mode=sq.SHARQ_MODE_NVFP4)
    es, en = H.rel_fro(ys, xw), H.rel_fro(yn, xw)
    assert es < 0.6 * en, (es, en)


def test_moe_grouped_matches_oracle():
    """Expert-sorted gather with 128-row padded groups + grouped GEMM."""
    K, D, E, T = 512, 256, 6, 300
    g = np.random.default_rng(12)
    x = synthetic.activations(12, T, K)
    counts = np.array([70, 0, 130, 5, 200, 95])
    token = np.concatenate([g.choice(T, c, replace=False) for c in counts])
    pad = -(-counts // 128) * 128
    offs = np.concatenate([[0], np.cumsum(pad)]).astype(np.int32)
    ri = np.full(offs[-1], -1, np.int32)
    start = 0
    for e in range(E):
        ri[offs[e]:offs[e] + counts[e]] = token[start:start + counts[e]]
        start += counts[e]
    ws = [synthetic.weights(40 + e, K, D) for e in range(E)]
    gamma = synthetic.gamma(13, K)
    xin = np.where(ri[:, None] >= 0, x[np.maximum(ri, 0)], 0).astype(np.float32)
    p = O.prep(xin, gamma, 1e-5)
    ref = O.linear_grouped(p, [O.pack_weight(w_) for w_ in ws], offs)
    act = sq.PreparedAct(len(ri), K)
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma), 1e-5, torch.from_numpy(ri).cuda())
    pw = sq.PackedWeight(torch.from_numpy(np.stack(ws)).to(torch.bfloat16).cuda())
    y = sq.linear(act, pw, out_dtype=torch.float32, group_offsets=torch.from_numpy(offs).cuda())
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    assert H.rel_fro(y, ref) < 1e-5


def test_full_size_q_proj_sampled():
    """The bench workload (Llama-3.1-8B q_proj, K = D = 4096, T = 128) in the
    same launch configuration: full prep bit-exact, Y on sampled columns."""
    T, K, D = 128, 4096, 4096
    x = synthetic.activations(1000, T, K)
    gamma = synthetic.gamma(1001, K)
    w = synthetic.weights(1002, K, D)
    y = _run(x, gamma, 1e-5, w)
    p = O.prep(x, gamma, 1e-5)
    q = O.pack_weight(w)
    cols = np.random.default_rng(0).choice(D, 64, replace=False)
    a = O.dequant_sparse(p) + O.dequant_residual(p)
    ref = (a @ q["w_t"][:, cols]) * (np.float64(p["s_g"]) * np.float64(q["s_w"]))
    assert H.rel_fro(y[:, cols], ref) < 1e-5
