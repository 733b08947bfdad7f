"""sharq_prep_silu_mul: the SwiGLU product fused into the down-projection
prep (GPU).

kasblo.com explainer, section 4 (fusing the preparation): the epilogues
before the preparation join the prep kernel; for the down projection of a
Llama-style MLP that is h = bf16(silu_bf16(gate) * up).  Checked against the
oracle bit for bit:
  - the kernel's SiLU on every finite bf16 input (65280 values, up = 1, h
    written out): the float32 fast path and its float64 fallback together
    must give the correctly rounded bf16 for all of them;
  - the prep of h on down-projection shapes (K = 14336) in the single-launch
    form (two runs per thread) and the wide form, with h stored and without
    (the wide quantizer forms h again), in the SharQ mode and a Table-5 mode;
  - Y of sharq_linear after it.
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


def _act(T, K, mode):
    act = sq.PreparedAct(T, K, mode)
    act.buf.fill_(0xAB)
    act.reset()
    return act


def test_silu_every_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[np.isfinite(v)]
    assert v.size == 255 * 256
    g = v.reshape(255, 256)
    u = np.ones_like(g)
    act = _act(255, 256, sq.SHARQ_MODE_SHARQ)
    h = torch.empty((255, 256), dtype=torch.bfloat16, device="cuda")
    act.prep_silu_mul(H.bf16_dev(g), H.bf16_dev(u), h, None, 1e-5)
    torch.cuda.synchronize()
    got = (h.view(torch.int16).cpu().numpy().astype(np.uint16).astype(np.uint32) << 16)
    want = O.silu_bf16(g).view(np.uint32)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} inputs differ, first g bits {[hex(int(g.view(np.uint32)[tuple(b)]) >> 16) for b in bad[:5]]}"


def _inputs(T, K, seed):
    g = synthetic.activations(seed, T, K) * np.float32(0.5)
    u = synthetic.activations(seed + 1, T, K, base="student_t")
    g[0, :8] = np.float32(-90.0)  # deep in the negative tail (float64 path)
    return g.astype(np.float32), u.astype(np.float32)


def _prep(g, u, mode, out):
    T, K = g.shape
    act = _act(T, K, mode)
    h = torch.empty((T, K), dtype=torch.bfloat16, device="cuda") if out else None
    act.prep_silu_mul(H.bf16_dev(g), H.bf16_dev(u), h, None, 1e-5)
    torch.cuda.synchronize()
    return act, h


@pytest.mark.parametrize("T,K,out", [(16, 14336, True), (1, 4096, True), (700, 14336, True), (700, 14336, False),
                                     (300, 4096, False)])
def test_silu_prep_matches_oracle(T, K, out):
    g, u = _inputs(T, K, 3100 + T)
    act, h = _prep(g, u, sq.SHARQ_MODE_SHARQ, out)
    hh = O.silu_mul(g, u)
    if out:
        assert np.array_equal(h.float().cpu().numpy().view(np.uint32), hh.view(np.uint32))
    p = O.prep(hh, None, 1e-5)
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
    for f, v in got.items():
        bad = np.argwhere(v[:T] != p[f])
        assert bad.size == 0, f"{f}: {len(bad)} mismatches, first {bad[:4].tolist()}"


@pytest.mark.parametrize("T,K", [(700, 14336), (16, 14336)])
def test_silu_prep_h_may_alias_up(T, K):
    """h written over up itself (the wide form's elementwise first pass and
    the single-launch form): h is still the SwiGLU product, and the prepared
    operands equal those of sharq_prep on it."""
    g, u = _inputs(T, K, 3150 + T)
    act = _act(T, K, sq.SHARQ_MODE_SHARQ)
    ud = H.bf16_dev(u)
    act.prep_silu_mul(H.bf16_dev(g), ud, ud, None, 1e-5)
    ref = _act(T, K, sq.SHARQ_MODE_SHARQ)
    hh = O.silu_mul(g, u)
    ref.prep(H.bf16_dev(hh), None, 1e-5)
    torch.cuda.synchronize()
    assert np.array_equal(ud.float().cpu().numpy().view(np.uint32), hh.view(np.uint32))
    n = ref.view.gmax_bits - 16 - ref.buf.data_ptr()   # operands and scales, not the per-row 1/rms scratch
    assert torch.equal(act.buf[:n], ref.buf[:n])


@pytest.mark.parametrize("T,K", [(16, 4096), (700, 8192)])
def test_silu_dense_dense_mode_equals_prep_of_h(T, K):
    g, u = _inputs(T, K, 3200 + T)
    act, _ = _prep(g, u, sq.SHARQ_MODE_DENSE_DENSE, False)
    ref = _act(T, K, sq.SHARQ_MODE_DENSE_DENSE)
    ref.prep(H.bf16_dev(O.silu_mul(g, u)), None, 1e-5)
    torch.cuda.synchronize()
    assert torch.equal(act.buf, ref.buf)


def test_linear_after_silu_prep():
    T, K, D = 64, 14336, 512
    g, u = _inputs(T, K, 3300)
    w = synthetic.weights(3301, K, D)
    act, _ = _prep(g, u, sq.SHARQ_MODE_SHARQ, False)
    ref = O.linear(O.prep(O.silu_mul(g, u), None, 1e-5), O.pack_weight(w))
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    ws = sq.Workspace(T, K, D)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    assert H.rel_fro(y.cpu().numpy(), ref) < 1e-5


def test_silu_prep_with_rmsnorm_and_empty_batch():
    """gamma applies to h like any prep input (bit-exact); T = 0 touches nothing."""
    T, K = 24, 2048
    g, u = _inputs(T, K, 3400)
    gamma = synthetic.gamma(3401, K)
    act = _act(T, K, sq.SHARQ_MODE_SHARQ)
    act.prep_silu_mul(H.bf16_dev(g), H.bf16_dev(u), None, H.bf16_dev(gamma), 1e-5)
    ref = _act(T, K, sq.SHARQ_MODE_SHARQ)
    ref.prep(H.bf16_dev(O.silu_mul(g, u)), H.bf16_dev(gamma), 1e-5)
    torch.cuda.synchronize()
    assert torch.equal(act.buf, ref.buf)
    empty = sq.PreparedAct(0, K, sq.SHARQ_MODE_SHARQ)
    empty.prep_silu_mul(None, None, None, None, 1e-5)
    empty.prep_residual(None, None, None, None, 1e-5)
    torch.cuda.synchronize()
