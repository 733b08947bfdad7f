"""Table-5 operand modes (Sparse only, Dense+Dense, Sparse+Sparse) vs the
oracle (GPU).

xllm-io review, section 5.3 (Table 5).  sharq_prep's outputs for each mode
must equal the oracle's bit for bit (masks, metadata, codes, scale bytes) in
the single-launch form and in the two-launch form (T * K beyond one
co-resident grid); sharq_linear's Y must match the oracle's float64 product
of the same operands within the float32 contract, in the persistent GEMM
with 256- and 128-wide tiles.
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


def _prep(x, gamma, eps, mode):
    T, K = x.shape
    act = sq.PreparedAct(T, K, mode)
    act.buf.fill_(0xAB)
    act.reset()
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma) if gamma is not None else None, eps)
    torch.cuda.synchronize()
    return act


def _eq(name, got, want):
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[:4].tolist()}"


def _get(act, name, tile_bytes, K):
    tiles = (act.view.Tp // 128) * (K // 256)
    return act.region(name, tiles * tile_bytes).cpu().numpy()


PREP_CASES = [(16, 256, True), (130, 512, False), (64, 14336, True), (700, 8192, True)]


@pytest.mark.parametrize("T,K,gam", PREP_CASES)
def test_dense_dense_prep_bit_exact(T, K, gam):
    x = synthetic.activations(800 + T, T, K)
    gamma = synthetic.gamma(801, K) if gam else None
    act = _prep(x, gamma, 1e-5, sq.SHARQ_MODE_DENSE_DENSE)
    p = O.prep_dense_dense(x, gamma, 1e-5)
    Tp = act.view.Tp
    assert act.view.meta is None and act.view.r_meta is None
    assert act.region("s_g", 4).view(torch.float32).item() == float(p["s_g"])
    _eq("b_codes", _layout.untile_codes(_get(act, "sp_codes", 16384, K), Tp, K)[:T], p["b_codes"])
    _eq("b_sf", _layout.untile_sf(_get(act, "sp_sf", 2048, K), Tp, K, 16)[:T], p["b_sf"])
    _eq("r_codes", _layout.untile_codes(_get(act, "r_codes", 16384, K), Tp, K)[:T], p["r_codes"])
    _eq("r_sf", _layout.untile_sf(_get(act, "r_sf", 2048, K), Tp, K, 16)[:T], p["r_sf"])


@pytest.mark.parametrize("T,K,gam", PREP_CASES)
def test_sparse_sparse_prep_bit_exact(T, K, gam):
    x = synthetic.activations(900 + T, T, K, base="student_t" if K > 10000 else "normal")
    gamma = synthetic.gamma(901, K) if gam else None
    act = _prep(x, gamma, 1e-5, sq.SHARQ_MODE_SPARSE_SPARSE)
    p = O.prep_sparse_sparse(x, gamma, 1e-5)
    Tp = act.view.Tp
    assert act.region("s_g", 4).view(torch.float32).item() == float(p["s_g"])
    _eq("meta", _layout.untile_meta(_get(act, "meta", 2048, K), Tp, K)[:T], p["meta"])
    _eq("sp_codes", _layout.untile_sp_codes(_get(act, "sp_codes", 8192, K), Tp, K)[:T], p["sp_codes"])
    _eq("sp_sf", _layout.untile_sf(_get(act, "sp_sf", 1024, K), Tp, K, 32)[:T], p["sp_sf"])
    _eq("r_meta", _layout.untile_meta(_get(act, "r_meta", 2048, K), Tp, K)[:T], p["r_meta"])
    _eq("r_sp_codes", _layout.untile_sp_codes(_get(act, "r_codes", 8192, K), Tp, K)[:T], p["r_sp_codes"])
    _eq("r_sp_sf", _layout.untile_sf(_get(act, "r_sf", 1024, K), Tp, K, 32)[:T], p["r_sp_sf"])


MODES = [("sparse_only", sq.SHARQ_MODE_SPARSE_ONLY, O.prep), ("dense_dense", sq.SHARQ_MODE_DENSE_DENSE,
                                                               O.prep_dense_dense),
         ("sparse_sparse", sq.SHARQ_MODE_SPARSE_SPARSE, O.prep_sparse_sparse)]


@pytest.mark.parametrize("name,mode,oprep", MODES, ids=[m[0] for m in MODES])
@pytest.mark.parametrize("T,K,D", [(16, 4096, 4096), (300, 1024, 512), (1024, 1024, 2048), (200, 768, 384)])
def test_mode_linear(name, mode, oprep, T, K, D):
    x = synthetic.activations(1000 + T, T, K)
    gamma = synthetic.gamma(1001, K)
    w = synthetic.weights(1002, K, D)
    ref = O.linear_mode(oprep(x, gamma, 1e-5), O.pack_weight(w), name)
    act = _prep(x, gamma, 1e-5, mode)
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    ws = sq.Workspace(T, K, D)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    e = H.rel_fro(y.cpu().numpy(), ref)
    assert e < 1e-5, e
