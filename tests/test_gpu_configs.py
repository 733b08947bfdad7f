"""Full-size parity for the workload configurations (GPU), on sampled outputs.

  config 3  Llama-3.1-8B MLP prefill: gate/up 4096 -> 14336 (RMSNorm), down
            14336 -> 4096 (Student-t input), T = 512
  config 4  Qwen3-30B-A3B experts: 128 experts, top-8 of T = 4096 tokens
            (Zipf(1.1) routing), gate/up 2048 -> 1536 and down 768 -> 2048,
            expert-sorted gather with 128-row padded groups
  config 5  Qwen2.5-7B decoder-layer linears: qkv 3584 -> 4608, o 3584 ->
            3584, gate+up 3584 -> 37888, down 18944 -> 3584, T = 64

The prepared activation is compared bit for bit on sampled rows (the oracle
quantizes those rows with the full tensor's PTS scale); Y is compared on
sampled output columns (and rows) against the oracle's float64 product of
the same quantized operands, at the float32 output tolerance.
"""
import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
import synthetic
from oracle import sharq as O
from tests import _layout
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def _pts(x, gamma):
    xn, _ = O.rmsnorm(x, gamma, EPS)
    return O.pts_scale(xn)[0]


def _check_rows(act, x, gamma, rows, s_g):
    """bit-exact prep outputs on the sampled rows"""
    T, K = act.T, act.K
    tiles = (act.view.Tp // 128) * (K // 256)
    get = lambda name, n: act.region(name, n).cpu().numpy()
    g_meta = _layout.untile_meta(get("meta", tiles * 2048), act.view.Tp, K)[rows]
    g_sp = _layout.untile_sp_codes(get("sp_codes", tiles * 8192), act.view.Tp, K)[rows]
    g_spsf = _layout.untile_sf(get("sp_sf", tiles * 1024), act.view.Tp, K, 32)[rows]
    g_rc = _layout.untile_codes(get("r_codes", tiles * 16384), act.view.Tp, K)[rows]
    g_rsf = _layout.untile_sf(get("r_sf", tiles * 2048), act.view.Tp, K, 16)[rows]
    p = O.prep(x[rows], gamma, EPS, s_g=s_g)
    for name, g, o in (("meta", g_meta, p["meta"]), ("sp_codes", g_sp, p["sp_codes"]),
                       ("sp_sf", g_spsf, p["sp_sf"]), ("r_codes", g_rc, p["r_codes"]), ("r_sf", g_rsf, p["r_sf"])):
        assert np.array_equal(g, o), name
    return p


def _check_y(y, p, w, cols, s_g):
    a = O.dequant_sparse(p) + O.dequant_residual(p)
    # weights quantize per output column with the whole weight's s_w: the
    # sampled columns are quantized exactly as pack_weight would
    s_w = np.float32(np.float32(np.max(np.abs(w))) / np.float32(2688))
    qw = O.nvfp4_quant(np.ascontiguousarray(w[:, cols].T).reshape(len(cols), -1, 32), s_w)
    from oracle.formats import e2m1_decode, e4m3_decode
    wt = (e2m1_decode(qw[0]) * e4m3_decode(qw[1])[..., None]).reshape(len(cols), -1).T
    ref = (a @ wt) * (np.float64(s_g) * np.float64(s_w))
    err = H.rel_fro(y, ref)
    assert err < 1e-5, err


def _run_linear(x, gamma, Ws, T):
    K = x.shape[1]
    act = sq.PreparedAct(T, K)
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma) if gamma is not None else None, EPS)
    ys = []
    for w in Ws:
        pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
        ys.append(sq.linear(act, pw, out_dtype=torch.float32))
    torch.cuda.synchronize()
    s_g = act.region("s_g", 4).view(torch.float32).item()
    return act, [y.cpu().numpy() for y in ys], s_g


@pytest.mark.parametrize("layer", ["gate_up", "down"])
def test_config3_llama_mlp_prefill(layer):
    T = 512
    g = np.random.default_rng(3)
    if layer == "gate_up":
        K, Ds = 4096, [14336, 14336]
        x = synthetic.activations(301, T, K)
        gamma = synthetic.gamma(302, K)
    else:
        K, Ds = 14336, [4096]
        x = synthetic.activations(303, T, K, base="student_t")
        gamma = None
    Ws = [synthetic.weights(310 + i, K, D) for i, D in enumerate(Ds)]
    act, ys, s_g = _run_linear(x, gamma, Ws, T)
    assert s_g == float(_pts(x, gamma))
    rows = np.sort(g.choice(T, 24, replace=False))
    p = _check_rows(act, x, gamma, rows, s_g)
    for w, y in zip(Ws, ys):
        cols = np.sort(g.choice(w.shape[1], 48, replace=False))
        _check_y(y[np.ix_(rows, cols)], p, w, cols, s_g)


@pytest.mark.parametrize("name,K,D,T,norm", [
    ("qkv", 3584, 4608, 64, True), ("o_proj", 3584, 3584, 64, False),
    ("gate_up", 3584, 37888, 64, True), ("down", 18944, 3584, 64, False)])
def test_config5_qwen_layer_linears(name, K, D, T, norm):
    g = np.random.default_rng(5)
    x = synthetic.activations(500 + K, T, K, base="normal" if name != "down" else "student_t")
    gamma = synthetic.gamma(501, K) if norm else None
    w = synthetic.weights(502 + D, K, D)
    act, (y,), s_g = _run_linear(x, gamma, [w], T)
    assert s_g == float(_pts(x, gamma))
    rows = np.sort(g.choice(T, 16, replace=False))
    p = _check_rows(act, x, gamma, rows, s_g)
    cols = np.sort(g.choice(D, 48, replace=False))
    _check_y(y[np.ix_(rows, cols)], p, w, cols, s_g)


def test_config4_qwen_moe_experts():
    """Zipf-routed top-8 of 4096 tokens over 128 experts, gate/up grouped
    GEMM (2048 -> 1536) on the expert-sorted, 128-padded gather, and the
    down projection (768 -> 2048) on a synthetic expert intermediate."""
    T, K, E, top = 4096, 2048, 128, 8
    tok, offs = synthetic.moe_routing(400, T, E, top)
    counts = np.diff(offs)
    pad = -(-counts // 128) * 128
    poffs = np.concatenate([[0], np.cumsum(pad)]).astype(np.int32)
    ri = np.full(int(poffs[-1]), -1, np.int32)
    for e in range(E):
        ri[poffs[e]:poffs[e] + counts[e]] = tok[offs[e]:offs[e + 1]]
    x = synthetic.activations(401, T, K, channel_frac=0.005)
    gamma = synthetic.gamma(402, K)
    g = np.random.default_rng(4)
    experts = np.sort(g.choice(np.nonzero(counts)[0], 3, replace=False))
    Wg = np.stack([synthetic.weights(410 + e, K, 1536) for e in range(E)])
    act = sq.PreparedAct(len(ri), K)
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma), EPS, torch.from_numpy(ri).cuda())
    pw = sq.PackedWeight(torch.from_numpy(Wg).to(torch.bfloat16).cuda())
    y = sq.linear(act, pw, out_dtype=torch.float32, group_offsets=torch.from_numpy(poffs).cuda())
    torch.cuda.synchronize()
    s_g = act.region("s_g", 4).view(torch.float32).item()
    xin = x[ri[ri >= 0]]
    assert s_g == float(_pts(xin, gamma))     # max over the gathered rows
    y = y.cpu().numpy()
    for e in experts:
        lo = int(poffs[e])
        rows = np.arange(lo, lo + min(int(counts[e]), 8))
        xr = x[ri[rows]]
        p = O.prep(xr, gamma, EPS, s_g=s_g)
        cols = np.sort(g.choice(1536, 32, replace=False))
        _check_y(y[np.ix_(rows, cols)], p, Wg[e], cols, s_g)
    # down projection of a synthetic expert intermediate, grouped the same way
    h = synthetic.activations(420, len(ri), 768, n_channels=4, channel_scale=(20.0, 60.0))
    Wd = np.stack([synthetic.weights(430 + e, 768, 2048) for e in range(E)])
    act2 = sq.PreparedAct(len(ri), 768)
    act2.prep(H.bf16_dev(h), None, EPS)
    pw2 = sq.PackedWeight(torch.from_numpy(Wd).to(torch.bfloat16).cuda())
    y2 = sq.linear(act2, pw2, out_dtype=torch.float32, group_offsets=torch.from_numpy(poffs).cuda())
    torch.cuda.synchronize()
    s2 = act2.region("s_g", 4).view(torch.float32).item()
    assert s2 == float(O.pts_scale(h)[0])
    y2 = y2.cpu().numpy()
    for e in experts:
        lo = int(poffs[e])
        rows = np.arange(lo, lo + min(int(counts[e]), 8))
        p = O.prep(h[rows], None, EPS, s_g=s2)
        cols = np.sort(g.choice(2048, 32, replace=False))
        _check_y(y2[np.ix_(rows, cols)], p, Wd[e], cols, s2)
