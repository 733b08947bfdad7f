"""Per-token global scales (SHARQ_MODE_SHARQ_TOKEN) vs the oracle (GPU).

Every row's s_t, mask, codes and scale bytes must equal the oracle's
per-token prep bit for bit; Y must match the oracle's float64 product of the
same quantized operands (each row scaled by its own s_t) within the float32
contract.  Covered: one and two runs per thread and four runs per thread
(K = 18944), grids far larger than the GPU (no device-wide reduction in this
mode), rows gathered with zero padding rows, the persistent and the split-K
GEMM, and the grouped expert form.
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

MODE = sq.SHARQ_MODE_SHARQ_TOKEN


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def _prep(x, gamma, eps, row_index=None):
    T = x.shape[0] if row_index is None else len(row_index)
    K = x.shape[1]
    act = sq.PreparedAct(T, K, MODE)
    act.buf.fill_(0xAB)
    act.reset()
    ri = torch.from_numpy(row_index.astype(np.int32)).cuda() if row_index is not None else None
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma) if gamma is not None else None, eps, ri)
    torch.cuda.synchronize()
    return act


def _check(act, T, K, p):
    Tp = act.view.Tp
    tiles = (Tp // 128) * (K // 256)
    get = lambda name, n: act.region(name, n).cpu().numpy()
    s_t = act.region("s_g", 4 * Tp).view(torch.float32).cpu().numpy()[:T]
    assert np.array_equal(s_t, p["s_g"])
    got = dict(
        meta=_layout.untile_meta(get("meta", tiles * 2048), Tp, K),
        sp_codes=_layout.untile_sp_codes(get("sp_codes", tiles * 8192), Tp, K),
        sp_sf=_layout.untile_sf(get("sp_sf", tiles * 1024), Tp, K, 32),
        r_codes=_layout.untile_codes(get("r_codes", tiles * 16384), Tp, K),
        r_sf=_layout.untile_sf(get("r_sf", tiles * 2048), Tp, K, 16),
    )
    for f, g in got.items():
        bad = np.argwhere(g[:T] != p[f])
        assert bad.size == 0, f"{f}: {len(bad)} mismatches, first {bad[:4].tolist()}"


@pytest.mark.parametrize("T,K,gam", [(16, 256, True), (130, 512, False), (64, 14336, True), (33, 18944, False),
                                     (1100, 1024, True)])
def test_per_token_prep_bit_exact(T, K, gam):
    x = synthetic.activations(500 + T, T, K, base="student_t" if K > 10000 else "normal")
    x[min(3, T - 1)] *= 64.0  # one dominant row: per-token and per-tensor codes differ
    gamma = synthetic.gamma(501, K) if gam else None
    act = _prep(x, gamma, 1e-5)
    _check(act, T, K, O.prep_per_token(x, gamma, 1e-5))


def test_per_token_gather_with_padding_rows():
    K = 512
    x = synthetic.activations(9, 40, K)
    ri = np.array(list(range(0, 40, 3)) + [-1] * 9 + list(range(1, 40, 5)), np.int32)
    act = _prep(x, synthetic.gamma(2, K), 1e-5, ri)
    xin = np.where(ri[:, None] >= 0, x[np.maximum(ri, 0)], 0).astype(np.float32)
    _check(act, len(ri), K, O.prep_per_token(xin, synthetic.gamma(2, K), 1e-5))


def test_per_token_differs_from_per_tensor():
    T, K = 8, 256
    x = synthetic.activations(3, T, K)
    x[2] *= 64.0
    a = _prep(x, None, 1e-5)
    b = sq.PreparedAct(T, K, sq.SHARQ_MODE_SHARQ)
    b.prep(H.bf16_dev(x), None, 1e-5)
    torch.cuda.synchronize()
    n = (K // 256) * 16384
    assert not torch.equal(a.region("r_codes", n), b.region("r_codes", n))


@pytest.mark.parametrize("T,K,D", [(16, 4096, 4096), (300, 1024, 512), (1024, 1024, 2048)])
def test_per_token_linear(T, K, D):
    """T=16: split-K decode GEMM; 300 and 1024: the persistent GEMM."""
    x = synthetic.activations(600 + T, T, K)
    x[min(5, T - 1)] *= 64.0
    gamma = synthetic.gamma(601, K)
    w = synthetic.weights(602, K, D)
    ref = O.linear(O.prep_per_token(x, gamma, 1e-5), O.pack_weight(w))
    act = _prep(x, gamma, 1e-5)
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    ws = sq.Workspace(T, K, D)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    e = H.rel_fro(y.cpu().numpy(), ref)
    assert e < 1e-5, e


def test_per_token_grouped_experts():
    K, D, E = 512, 256, 3
    counts = [128, 0, 256]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    T = int(offsets[-1])
    x = synthetic.activations(77, T, K)
    ws_ = [synthetic.weights(80 + e, K, D) for e in range(E)]
    ref = O.linear_grouped(O.prep_per_token(x, None, 1e-5), [O.pack_weight(w) for w in ws_], offsets)
    act = _prep(x, None, 1e-5)
    pw = sq.PackedWeight(torch.from_numpy(np.stack(ws_)).to(torch.bfloat16).cuda())
    ws = sq.Workspace(T, K, D, E)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws, group_offsets=torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    assert ws.check() == 0
    assert H.rel_fro(y.cpu().numpy(), ref) < 1e-5
