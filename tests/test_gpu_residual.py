"""sharq_prep_residual: the residual-stream update fused into the prep (GPU).

kasblo.com explainer, section 4 (fusing the preparation): the epilogues that
come before RMSNorm join the preparation kernel.  For a pre-norm layer that
epilogue is h = x + res.  The prep of sharq_prep_residual(x, res) must equal
the oracle's prep of h = residual_add(x, res) bit for bit, and the updated
stream it writes must equal residual_add(x, res) bit for bit.  Covered: every
load site of the prep (single launch with 1, 2 and 4 runs per thread; the wide
form's row statistics with and without RMSNorm, its strip quantizer and its
runs quantizer), every operand mode, rows that cancel to zero, the in-place
update (res_out == res) and the form that does not store h.
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def _inputs(T, K, seed):
    x = synthetic.activations(seed, T, K, base="student_t" if K > 10000 else "normal")
    r = synthetic.activations(seed + 1, T, K, n_channels=4, channel_scale=(40.0, 120.0)) * np.float32(4.0)
    r[0] = -x[0]  # a row that cancels to exactly zero
    return x, r.astype(np.float32)


def _act(T, K, mode):
    act = sq.PreparedAct(T, K, mode)
    act.buf.fill_(0xAB)
    act.reset()
    return act


def _prep_residual(x, r, gamma, eps, mode, out="new"):
    T, K = x.shape
    act = _act(T, K, mode)
    X, R = H.bf16_dev(x), H.bf16_dev(r)
    Hout = {"new": torch.full_like(R, float("nan")), "inplace": R, "none": None}[out]
    act.prep_residual(X, R, Hout, H.bf16_dev(gamma) if gamma is not None else None, eps)
    torch.cuda.synchronize()
    return act, R, Hout


def _check_h(got, x, r):
    want = O.residual_add(x, r)
    g = got.float().cpu().numpy()
    bad = np.argwhere(g.view(np.uint32) != want.view(np.uint32))
    assert bad.size == 0, f"h: {len(bad)} mismatches, first {bad[:4].tolist()}"


# (T, K, gamma): single launch with 1, 2, 4 runs per thread; the wide form
# with RMSNorm (strip quantizer) and without (rows of the statistics kernel
# that only take max |h|)
SHARQ_CASES = [(1, 256, True), (16, 4096, True), (64, 14336, True), (33, 18944, False), (700, 8192, True),
               (600, 4096, False)]


@pytest.mark.parametrize("T,K,gam", SHARQ_CASES)
def test_residual_prep_matches_oracle(T, K, gam):
    x, r = _inputs(T, K, 1300 + T)
    gamma = synthetic.gamma(1301, K) if gam else None
    act, _, h = _prep_residual(x, r, gamma, 1e-5, sq.SHARQ_MODE_SHARQ)
    _check_h(h, x, r)
    p = O.prep(O.residual_add(x, r), gamma, 1e-5)
    Tp = act.view.Tp
    tiles = (Tp // 128) * (K // 256)
    get = lambda name, n: act.region(name, n).cpu().numpy()
    assert act.region("s_g", 4).view(torch.float32).item() == float(p["s_g"])
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
    # the row that cancelled is a zero row: nothing kept, nothing coded
    assert not got["sp_codes"][0].any() and not got["r_codes"][0].any()


MODES = [sq.SHARQ_MODE_SHARQ, sq.SHARQ_MODE_NVFP4, sq.SHARQ_MODE_SHARQ_TOKEN, sq.SHARQ_MODE_SPARSE_ONLY,
         sq.SHARQ_MODE_DENSE_DENSE, sq.SHARQ_MODE_SPARSE_SPARSE, sq.SHARQ_MODE_MXFP4, sq.SHARQ_MODE_MXFP4_PLAIN]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("T,K", [(16, 4096), (700, 8192)])
def test_residual_every_mode_equals_prep_of_h(mode, T, K):
    """The whole prepared buffer equals sharq_prep's on the oracle's h (whose
    parity with the oracle's prep the per-mode tests establish)."""
    x, r = _inputs(T, K, 1400 + T)
    gamma = synthetic.gamma(1401, K)
    act, _, h = _prep_residual(x, r, gamma, 1e-5, mode)
    _check_h(h, x, r)
    ref = _act(T, K, mode)
    ref.prep(H.bf16_dev(O.residual_add(x, r)), H.bf16_dev(gamma), 1e-5)
    torch.cuda.synchronize()
    diff = (act.buf != ref.buf).nonzero()
    assert diff.numel() == 0, f"{diff.numel()} bytes differ, first at {diff[:4].flatten().tolist()}"


@pytest.mark.parametrize("T,K", [(16, 4096), (700, 8192)])
def test_in_place_update(T, K):
    x, r = _inputs(T, K, 1500 + T)
    gamma = synthetic.gamma(1501, K)
    act, R, _ = _prep_residual(x, r, gamma, 1e-5, sq.SHARQ_MODE_SHARQ, out="inplace")
    _check_h(R, x, r)
    ref = _act(T, K, sq.SHARQ_MODE_SHARQ)
    ref.prep(H.bf16_dev(O.residual_add(x, r)), H.bf16_dev(gamma), 1e-5)
    torch.cuda.synchronize()
    assert torch.equal(act.buf, ref.buf)


@pytest.mark.parametrize("T,K,gam,mode", [(40, 2048, False, sq.SHARQ_MODE_SHARQ),
                                          (700, 8192, True, sq.SHARQ_MODE_SHARQ),
                                          (600, 4096, False, sq.SHARQ_MODE_SHARQ),
                                          (700, 8192, True, sq.SHARQ_MODE_DENSE_DENSE)])
def test_without_stream_output(T, K, gam, mode):
    """h not stored: the wide form's quantizer forms h again from x and res."""
    x, r = _inputs(T, K, 1600 + T)
    gamma = synthetic.gamma(1601, K) if gam else None
    act, R, _ = _prep_residual(x, r, gamma, 1e-5, mode, out="none")
    assert torch.equal(R, H.bf16_dev(r))  # the input stream is left as it was
    ref = _act(T, K, mode)
    ref.prep(H.bf16_dev(O.residual_add(x, r)), H.bf16_dev(gamma) if gam else None, 1e-5)
    torch.cuda.synchronize()
    assert torch.equal(act.buf, ref.buf)


def test_linear_after_residual_prep():
    """Y of sharq_linear on the residual prep equals the oracle's GEMM of the
    oracle's prep of h."""
    T, K, D = 48, 4096, 1024
    x, r = _inputs(T, K, 1700)
    gamma = synthetic.gamma(1701, K)
    w = synthetic.weights(1702, K, D)
    act, _, _ = _prep_residual(x, r, gamma, 1e-5, sq.SHARQ_MODE_SHARQ)
    ref = O.linear(O.prep(O.residual_add(x, r), gamma, 1e-5), O.pack_weight(w))
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    ws = sq.Workspace(T, K, D)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    assert H.rel_fro(y.cpu().numpy(), ref) < 1e-5


def test_argument_errors():
    T, K = 8, 256
    act = _act(T, K, sq.SHARQ_MODE_SHARQ)
    X = torch.zeros((T, K), dtype=torch.bfloat16, device="cuda")
    R = torch.zeros_like(X)
    with pytest.raises(sq.SharqError):  # the updated stream may not overwrite X
        sq.sharq_prep_residual(X.data_ptr(), R.data_ptr(), X.data_ptr(), None, 1e-5, act.view, None)
    with pytest.raises(sq.SharqError):  # no residual stream
        sq.sharq_prep_residual(X.data_ptr(), None, None, None, 1e-5, act.view, None)
    with pytest.raises(sq.SharqError):  # misaligned residual stream
        sq.sharq_prep_residual(X.data_ptr(), R.data_ptr() + 2, None, None, 1e-5, act.view, None)
    torch.cuda.synchronize()
