"""Full-size parity of the workload configurations over their whole T sweeps
(GPU), every row compared.

  config 3  Llama-3.1-8B MLP prefill, T = 2048 and 8192: gate and up
            (4096 -> 14336 each, one shared RMSNorm prep), down 14336 -> 4096
            (Student-t input)
  config 5  Qwen2.5-7B decoder-layer linears, T = 1, 64, 1024 and 8192: qkv
            3584 -> 4608 and gate+up 3584 -> 37888 (RMSNorm), o 3584 -> 3584,
            down 18944 -> 3584 (Student-t input)
  config 4  Qwen3-30B-A3B experts: every expert with a non-empty group, every
            m-tile of every group

The prepared activation (metadata, backbone codes and scales, residual codes
and scales) is compared bit for bit on every row against the oracle, which
prepares row chunks in parallel with the whole tensor's per-tensor scale.  Y
(float32 output mode) is compared on every row and on one random column of
every 128-column group, so every output tile that the persistent scheduler
visits -- including the later tiles of each CTA, whose stage-ring phases run
on from earlier tiles -- is checked; each (128-row, 256-column) block must be
within 1e-5 relative Frobenius error of the oracle's float64 product of the
same quantized operands (the contract allows 1e-3).
"""
import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
import synthetic
from tests import _layout
from tests import _oracle_pool as P
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
EPS = 1e-5
Y_TOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()
    P.pool()    # spawn the oracle workers up front


def _gpu_operands(act):
    T, K, Tp = act.T, act.K, act.view.Tp
    tiles = (Tp // 128) * (K // 256)
    get = lambda name, n: act.region(name, n).cpu().numpy()
    return {"meta": _layout.untile_meta(get("meta", tiles * 2048), Tp, K)[:T],
            "sp_codes": _layout.untile_sp_codes(get("sp_codes", tiles * 8192), Tp, K)[:T],
            "sp_sf": _layout.untile_sf(get("sp_sf", tiles * 1024), Tp, K, 32)[:T],
            "r_codes": _layout.untile_codes(get("r_codes", tiles * 16384), Tp, K)[:T],
            "r_sf": _layout.untile_sf(get("r_sf", tiles * 2048), Tp, K, 16)[:T]}


def _compare_operands(got, ref, where):
    for name in ("meta", "sp_codes", "sp_sf", "r_codes", "r_sf"):
        g, o = got[name], ref[name]
        assert g.shape == o.shape, (where, name, g.shape, o.shape)
        bad = np.nonzero(np.any((g != o).reshape(len(g), -1), axis=1))[0]
        assert bad.size == 0, f"{where}: {name} differs on {bad.size} rows, first {bad[:8].tolist()}"


def _compare_y(y, ref, cols, row_blocks, where):
    """y, ref: [rows, len(cols)]; cols sorted, one per 128-column group.
    row_blocks: list of (lo, hi) row ranges (the m-tiles)."""
    groups = cols // 256
    worst = 0.0
    for lo, hi in row_blocks:
        for nt in np.unique(groups):
            sel = groups == nt
            e = H.rel_fro(y[lo:hi][:, sel], ref[lo:hi][:, sel])
            worst = max(worst, e)
            assert e < Y_TOL, f"{where}: rows {lo}:{hi}, n-tile {nt}: rel_fro {e:.3e}"
    return worst


def _cols(g, D):
    return np.array([128 * j + int(g.integers(0, 128)) for j in range(D // 128)])


def _chunk(K):
    return 128 if K >= 8192 else 512


def _run_layer(x, gamma, Ws, where, seed):
    """prep on the GPU, sharq_linear for each weight (float32 out); compare
    every row of the operands and sampled columns of every Y tile."""
    T, K = x.shape
    g = np.random.default_rng(seed)
    act = sq.PreparedAct(T, K)
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma) if gamma is not None else None, EPS)
    cols, ys = [], []
    for w in Ws:
        pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
        y = sq.linear(act, pw, out_dtype=torch.float32)
        c = _cols(g, w.shape[1])
        ys.append(y[:, torch.from_numpy(c).cuda()].cpu().numpy())
        cols.append(c)
        del pw, y
    torch.cuda.synchronize()
    s_g = act.region("s_g", 4).view(torch.float32).item()
    got = _gpu_operands(act)
    del act
    chunk = _chunk(K)
    assert s_g == float(P.tensor_scale(x, gamma, EPS, chunk)), where
    ref = P.prep_all(x, gamma, EPS, np.float32(s_g), [P.sampled_weight(w, c) for w, c in zip(Ws, cols)], chunk)
    _compare_operands(got, ref, where)
    blocks = [(lo, min(lo + 128, T)) for lo in range(0, T, 128)]
    for j, (y, c) in enumerate(zip(ys, cols)):
        _compare_y(y, ref["y"][j], c, blocks, f"{where} weight {j}")


@pytest.mark.parametrize("T", [2048, 8192])
@pytest.mark.parametrize("layer", ["gate_up", "down"])
def test_config3_llama_mlp_full(layer, T):
    if layer == "gate_up":
        K = 4096
        x = synthetic.activations(3100 + T, T, K)
        gamma = synthetic.gamma(3101, K)
        Ws = [synthetic.weights(3110 + i, K, 14336) for i in range(2)]
    else:
        K = 14336
        x = synthetic.activations(3200 + T, T, K, base="student_t")
        gamma = None
        Ws = [synthetic.weights(3210, K, 4096)]
    _run_layer(x, gamma, Ws, f"config3 {layer} T={T}", 30 + T)


QWEN = {"qkv": (3584, 4608, True), "o_proj": (3584, 3584, False), "gate_up": (3584, 37888, True),
        "down": (18944, 3584, False)}


@pytest.mark.parametrize("T", [1, 64, 1024, 8192])
@pytest.mark.parametrize("name", list(QWEN))
def test_config5_qwen_layer_full(name, T):
    K, D, norm = QWEN[name]
    x = synthetic.activations(5100 + T + K, T, K, base="student_t" if name == "down" else "normal")
    gamma = synthetic.gamma(5101, K) if norm else None
    Ws = [synthetic.weights(5110 + D, K, D)]
    _run_layer(x, gamma, Ws, f"config5 {name} T={T}", 50 + T)


def _moe_gather(T, E, top):
    tok, offs = synthetic.moe_routing(400, T, E, top)
    counts = np.diff(offs)
    pad = -(-counts // 128) * 128
    poffs = np.concatenate([[0], np.cumsum(pad)]).astype(np.int32)
    ri = np.full(int(poffs[-1]), -1, np.int32)
    for e in range(E):
        ri[poffs[e]:poffs[e] + counts[e]] = tok[offs[e]:offs[e + 1]]
    return ri, counts, poffs


def _grouped_check(a_in, gamma, ri, counts, poffs, Ws, where):
    """Grouped GEMM over E experts.  With gamma, a_in is the token tensor and
    sharq_prep gathers the expert-sorted rows by ri (zero rows where ri < 0);
    without, a_in already holds the rows in expert order.  Every row of every
    group (padding rows included) is compared, and Y on the group's token
    rows, every m-tile."""
    E = len(Ws)
    g = np.random.default_rng(44)
    rows_total, K = len(ri), Ws[0].shape[0]
    D = Ws[0].shape[1]
    act = sq.PreparedAct(rows_total, K)
    if gamma is not None:
        act.prep(H.bf16_dev(a_in), H.bf16_dev(gamma), EPS, torch.from_numpy(ri).cuda())
        xg = np.where(ri[:, None] >= 0, a_in[np.maximum(ri, 0)], np.float32(0)).astype(np.float32)
    else:
        act.prep(H.bf16_dev(a_in), None, EPS)
        xg = a_in
    pw = sq.PackedWeight(torch.from_numpy(np.stack(Ws)).to(torch.bfloat16).cuda())
    y = sq.linear(act, pw, out_dtype=torch.float32, group_offsets=torch.from_numpy(poffs).cuda())
    c = _cols(g, D)
    y = y[:, torch.from_numpy(c).cuda()].cpu().numpy()
    torch.cuda.synchronize()
    s_g = act.region("s_g", 4).view(torch.float32).item()
    got = _gpu_operands(act)
    del act, pw
    # the per-tensor scale is over the gathered rows (zero padding rows add 0)
    assert s_g == float(P.tensor_scale(xg, gamma, EPS, 1024)), where
    groups = [e for e in range(E) if poffs[e + 1] > poffs[e]]
    jobs = [(xg[poffs[e]:poffs[e + 1]], gamma, EPS, np.float32(s_g), [P.sampled_weight(Ws[e], c)]) for e in groups]
    res = P.pool().map(P.prep_rows, jobs)
    for e, r in zip(groups, res):
        lo, hi, n = int(poffs[e]), int(poffs[e + 1]), int(counts[e])
        _compare_operands({k: v[lo:hi] for k, v in got.items()}, r, f"{where} expert {e}")
        blocks = [(b, min(b + 128, n)) for b in range(0, n, 128)]
        _compare_y(y[lo:lo + n], r["y"][0][:n], c, blocks, f"{where} expert {e}")
    assert sum(poffs[e + 1] - poffs[e] for e in groups) == rows_total


def test_config4_qwen_moe_full():
    """Every non-empty expert group and every m-tile of it: gate/up
    (2048 -> 1536) on the Zipf-routed, expert-sorted gather of 4096 tokens
    x top-8, and the down projection (768 -> 2048) on a synthetic expert
    intermediate of the same row layout."""
    T, K, E, top = 4096, 2048, 128, 8
    ri, counts, poffs = _moe_gather(T, E, top)
    assert counts.max() > 256          # the largest groups span several m-tiles
    x = synthetic.activations(401, T, K, channel_frac=0.005)
    gamma = synthetic.gamma(402, K)
    Wg = [synthetic.weights(4410 + e, K, 1536) for e in range(E)]
    _grouped_check(x, gamma, ri, counts, poffs, Wg, "config4 gate_up")
    h = synthetic.activations(420, len(ri), 768, n_channels=4, channel_scale=(20.0, 60.0))
    Wd = [synthetic.weights(4430 + e, 768, 2048) for e in range(E)]
    _grouped_check(h, None, ri, counts, poffs, Wd, "config4 down")
