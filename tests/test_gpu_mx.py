"""MXFP4 variant (SHARQ_MODE_MXFP4, SHARQ_MODE_MXFP4_PLAIN, SHARQ_FMT_MXFP4)
vs the oracle (GPU).

xllm-io review, section 5.3 (SharQ across NVFP4, HiF4 and MXFP4); MXFP4 as
defined by the OCP Microscaling Formats specification (E2M1 elements, E8M0
power-of-two block scales).  The packed weight and the prepared activation
must equal the oracle's bit for bit (codes, masks, metadata, E8M0 bytes), in
the single-launch and the two-launch prep forms; Y must match the oracle's
float64 product of the same operands within the float32 contract (the
kind::mxf4 sparse and dense MMAs of the persistent GEMM, 256- and 128-wide
tiles).
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


def _eq(name, got, want):
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[:4].tolist()}"


def _prep(x, gamma, mode):
    T, K = x.shape
    act = sq.PreparedAct(T, K, mode)
    act.buf.fill_(0xAB)
    act.reset()
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma) if gamma is not None else None, 1e-5)
    torch.cuda.synchronize()
    return act


def _get(act, name, tile_bytes, K):
    tiles = (act.view.Tp // 128) * (K // 256)
    return act.region(name, tiles * tile_bytes).cpu().numpy()


@pytest.mark.parametrize("K,D", [(256, 256), (512, 384), (4096, 128)])
def test_pack_weight_mx_bit_exact(K, D):
    w = synthetic.weights(40 + K, K, D)
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda(), fmt=sq.SHARQ_FMT_MXFP4)
    torch.cuda.synchronize()
    q = O.pack_weight_mx(w)
    tiles = (D // 128) * (K // 256)
    base = pw.buf.data_ptr()
    get = lambda ptr, n: pw.buf[ptr - base:ptr - base + n].cpu().numpy()
    _eq("codes", _layout.untile_codes(get(pw.view.codes, tiles * 16384), D, K), q["codes"])
    _eq("sf64", _layout.untile_sf(get(pw.view.sf32, tiles * 512), D, K, 64), q["sf64"])
    _eq("sf32", _layout.untile_sf(get(pw.view.sf16, tiles * 1024), D, K, 32), q["sf32"])
    assert pw.s_w().item() == 1.0


PREP_CASES = [(16, 256, True), (130, 512, False), (64, 14336, True), (700, 8192, True)]


@pytest.mark.parametrize("T,K,gam", PREP_CASES)
def test_prep_mx_bit_exact(T, K, gam):
    x = synthetic.activations(1100 + T, T, K, base="student_t" if K > 10000 else "normal")
    gamma = synthetic.gamma(1101, K) if gam else None
    act = _prep(x, gamma, sq.SHARQ_MODE_MXFP4)
    p = O.prep_mxfp4(x, gamma, 1e-5)
    Tp = act.view.Tp
    assert act.region("s_g", 4).view(torch.float32).item() == 1.0
    _eq("meta", _layout.untile_meta(_get(act, "meta", 2048, K), Tp, K)[:T], p["meta"])
    _eq("sp_codes", _layout.untile_sp_codes(_get(act, "sp_codes", 8192, K), Tp, K)[:T], p["sp_codes"])
    _eq("sp_sf", _layout.untile_sf(_get(act, "sp_sf", 512, K), Tp, K, 64)[:T], p["sp_sf"])
    _eq("r_codes", _layout.untile_codes(_get(act, "r_codes", 16384, K), Tp, K)[:T], p["r_codes"])
    _eq("r_sf", _layout.untile_sf(_get(act, "r_sf", 1024, K), Tp, K, 32)[:T], p["r_sf"])


@pytest.mark.parametrize("T,K", [(16, 256), (700, 8192)])
def test_prep_mx_plain_bit_exact(T, K):
    x = synthetic.activations(1200 + T, T, K)
    gamma = synthetic.gamma(1201, K)
    act = _prep(x, gamma, sq.SHARQ_MODE_MXFP4_PLAIN)
    p = O.prep_mxfp4_plain(x, gamma, 1e-5)
    Tp = act.view.Tp
    _eq("codes", _layout.untile_codes(_get(act, "r_codes", 16384, K), Tp, K)[:T], p["codes"])
    _eq("sf", _layout.untile_sf(_get(act, "r_sf", 1024, K), Tp, K, 32)[:T], p["sf"])


@pytest.mark.parametrize("mode", [sq.SHARQ_MODE_MXFP4, sq.SHARQ_MODE_MXFP4_PLAIN], ids=["sharq_mx", "plain_mx"])
@pytest.mark.parametrize("T,K,D", [(16, 4096, 4096), (300, 1024, 512), (200, 768, 384)])
def test_linear_mx(mode, T, K, D):
    x = synthetic.activations(1300 + T, T, K)
    gamma = synthetic.gamma(1301, K)
    w = synthetic.weights(1302, K, D)
    p = O.prep_mxfp4(x, gamma, 1e-5) if mode == sq.SHARQ_MODE_MXFP4 else O.prep_mxfp4_plain(x, gamma, 1e-5)
    ref = O.linear_mx(p, O.pack_weight_mx(w))
    act = _prep(x, gamma, mode)
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda(), fmt=sq.SHARQ_FMT_MXFP4)
    ws = sq.Workspace(T, K, D)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    e = H.rel_fro(y.cpu().numpy(), ref)
    assert e < 1e-5, e


def test_format_mismatch_is_rejected():
    T, K, D = 16, 256, 256
    act = sq.PreparedAct(T, K, sq.SHARQ_MODE_MXFP4)
    pw = sq.PackedWeight(torch.zeros(K, D, dtype=torch.bfloat16, device="cuda"))  # NVFP4 payload
    with pytest.raises(sq.SharqError):
        sq.linear(act, pw, ws=sq.Workspace(T, K, D))
