"""sharq_prep and sharq_pack_weight vs the oracle, bit for bit (GPU).

Masks, metadata nibbles, E2M1 codes, E4M3 scale bytes and the FP32 global
scales must be identical on every row T of the tensor (the tile padding rows
past T are not part of the output).
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


def _gpu_prep(x, gamma, eps, mode=sq.SHARQ_MODE_SHARQ, row_index=None, T=None):
    T = x.shape[0] if T is None else T
    K = x.shape[1]
    act = sq.PreparedAct(T, K, mode)
    act.buf.fill_(0xAB)    # canary: every byte the layout defines must be written
    act.reset()            # ... except the scalar block, zero before first use
    xd = H.bf16_dev(x)
    gd = H.bf16_dev(gamma) if gamma is not None else None
    ri = torch.from_numpy(row_index.astype(np.int32)).cuda() if row_index is not None else None
    act.prep(xd, gd, eps, ri)
    torch.cuda.synchronize()
    return act


def _read(act, T, K, mode):
    Tp = act.view.Tp
    tiles = (Tp // 128) * (K // 256)
    get = lambda name, n: act.region(name, n).cpu().numpy()
    out = dict(
        s_g=act.region("s_g", 4).view(torch.float32).item(),
        r_codes=_layout.untile_codes(get("r_codes", tiles * 16384), Tp, K),
        r_sf=_layout.untile_sf(get("r_sf", tiles * 2048), Tp, K, 16),
    )
    if mode == sq.SHARQ_MODE_SHARQ:
        out["sp_codes"] = _layout.untile_sp_codes(get("sp_codes", tiles * 8192), Tp, K)
        out["meta"] = _layout.untile_meta(get("meta", tiles * 2048), Tp, K)
        out["sp_sf"] = _layout.untile_sf(get("sp_sf", tiles * 1024), Tp, K, 32)
    return out


def _assert_equal(name, got, want):
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{name}: {len(bad)} mismatches, first at {bad[:5].tolist()} " \
                          f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}"


def _check_sharq(x, gamma, eps, row_index=None, T=None):
    T = x.shape[0] if T is None else T
    K = x.shape[1]
    act = _gpu_prep(x, gamma, eps, row_index=row_index, T=T)
    g = _read(act, T, K, sq.SHARQ_MODE_SHARQ)
    xin = x if row_index is None else np.where(row_index[:, None] >= 0, x[np.maximum(row_index, 0)], 0)
    p = O.prep(xin.astype(np.float32), gamma, eps)
    assert g["s_g"] == float(p["s_g"])
    _assert_equal("meta", g["meta"][:T], p["meta"])
    _assert_equal("sp_codes", g["sp_codes"][:T], p["sp_codes"])
    _assert_equal("sp_sf", g["sp_sf"][:T], p["sp_sf"])
    _assert_equal("r_codes", g["r_codes"][:T], p["r_codes"])
    _assert_equal("r_sf", g["r_sf"][:T], p["r_sf"])
    return act, p


CASES = [
    # (name, T, K, activation kwargs, gamma, eps)
    ("single_linear_T16_K256", 16, 256, dict(n_channels=4, channel_scale=(30.0, 30.0), spike_p=0.01), "one", 1e-5),
    ("q_proj_T1_K4096", 1, 4096, dict(), "uniform", 1e-5),
    ("q_proj_T128_K4096", 128, 4096, dict(), "uniform", 1e-5),
    ("ragged_T130_K512", 130, 512, dict(), "uniform", 1e-6),
    ("down_student_t_T77_K768", 77, 768, dict(base="student_t", channel_frac=0.005), None, 1e-5),
]


@pytest.mark.parametrize("name,T,K,kw,gam,eps", CASES, ids=[c[0] for c in CASES])
def test_prep_bit_exact(name, T, K, kw, gam, eps):
    x = synthetic.activations(100 + T, T, K, **kw)
    gamma = None if gam is None else (synthetic.gamma(7, K, 1.0, 1.0) if gam == "one" else synthetic.gamma(8, K))
    _check_sharq(x, gamma, eps)


@pytest.mark.parametrize("T", [2, 9, 17])
def test_prep_grid_forms_bit_exact(T):
    """K = 4096 (one row per 512-thread CTA): T = 2 and 9 run as one
    thread-block cluster (9 is above the portable cluster size), T = 17 as a
    grid with the global-memory barrier."""
    K = 4096
    x = synthetic.activations(150 + T, T, K)
    x[T - 1] *= 32.0  # the tensor max in the last CTA
    _check_sharq(x, synthetic.gamma(151, K), 1e-5)


@pytest.mark.parametrize("T,K", [(64, 14336), (32, 18944), (33, 3584)])
def test_prep_long_rows_bit_exact(T, K):
    """Rows longer than 8192 give each thread 2 or 4 runs of 8 in the
    single-launch form (Llama MLP down_proj K = 14336, Qwen2.5-7B down_proj
    K = 18944, Qwen2.5-7B hidden 3584)."""
    x = synthetic.activations(77 + T, T, K, base="student_t")
    _check_sharq(x, synthetic.gamma(78, K), 1e-6)


@pytest.mark.parametrize("T,K", [(400, 14336), (700, 8192)])
def test_prep_two_launch_path_bit_exact(T, K):
    """Tensors too large for one co-resident grid take the two-launch form
    (stats kernel + quantize kernel); it must agree bit for bit as well."""
    x = synthetic.activations(55 + T, T, K, base="student_t" if K > 10000 else "normal")
    _check_sharq(x, synthetic.gamma(56, K), 1e-5)


def test_prep_nvfp4_mode_bit_exact():
    T, K = 130, 512
    x = synthetic.activations(5, T, K)
    gamma = synthetic.gamma(6, K)
    act = _gpu_prep(x, gamma, 1e-5, mode=sq.SHARQ_MODE_NVFP4)
    g = _read(act, T, K, sq.SHARQ_MODE_NVFP4)
    p = O.prep_nvfp4(x, gamma, 1e-5)
    assert g["s_g"] == float(p["s_g"])
    _assert_equal("codes", g["r_codes"][:T], p["codes"])
    _assert_equal("sf", g["r_sf"][:T], p["sf"])


def test_prep_edge_cases():
    K = 256
    # worked example row (one outlier among 0.2s), a zero row, a constant row,
    # rows at E2M1 rounding ties
    x = np.full((6, K), 0.2001953125, np.float32)
    x[0, 0] = 12.0
    x[1] = 0.0
    x[2] = -3.0
    x[3, ::2] = 0.25
    x[3, 1::2] = -0.75
    x[4] = np.tile(np.array([6, 5, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25], np.float32), K // 8)
    x[5, :] = np.float32(2.0 ** -20)
    _check_sharq(x, None, 1e-5)
    _check_sharq(x, synthetic.gamma(1, K), 1e-6)


def test_prep_gather_with_padding_rows():
    K = 512
    x = synthetic.activations(9, 50, K)
    ri = np.array(list(range(0, 50, 3)) + [-1] * 20 + list(range(1, 50, 7)), np.int32)
    _check_sharq(x, synthetic.gamma(2, K), 1e-5, row_index=ri, T=len(ri))


def test_prep_all_zero_tensor_and_empty():
    K = 256
    x = np.zeros((3, K), np.float32)
    act, p = _check_sharq(x, None, 1e-5)
    assert p["s_g"] == 1.0
    act = sq.PreparedAct(0, K)
    act.prep(None, None, 1e-5)
    torch.cuda.synchronize()
    assert act.region("s_g", 4).view(torch.float32).item() == 1.0


@pytest.mark.parametrize("K,D,E", [(256, 256, 1), (512, 384, 2), (4096, 128, 1)])
def test_pack_weight_bit_exact(K, D, E):
    ws = [synthetic.weights(30 + e, K, D) for e in range(E)]
    W = torch.from_numpy(np.stack(ws)).to(torch.bfloat16).cuda()
    pw = sq.PackedWeight(W if E > 1 else W[0])
    torch.cuda.synchronize()
    base = pw.buf.data_ptr()
    tiles = (D // 128) * (K // 256)
    buf = pw.buf.cpu().numpy()

    def region(ptr, n):
        return buf[ptr - base: ptr - base + n]
    for e in range(E):
        q = O.pack_weight(ws[e])
        codes = _layout.untile_codes(region(pw.view.codes + e * tiles * 16384, tiles * 16384), D, K)
        sf32 = _layout.untile_sf(region(pw.view.sf32 + e * tiles * 1024, tiles * 1024), D, K, 32)
        sf16 = _layout.untile_sf(region(pw.view.sf16 + e * tiles * 2048, tiles * 2048), D, K, 16)
        _assert_equal("w codes", codes, q["codes"])
        _assert_equal("w sf32", sf32, q["sf32"])
        _assert_equal("w sf16", sf16, q["sf16"])
        assert pw.s_w()[e].item() == float(q["s_w"])


@pytest.mark.parametrize("case", ["plain", "huge_gamma_on_zero_column", "mixed"])
def test_wide_rowstats_edge_rows(case):
    """The wide form (statistics launch, then the strip quantizer) against the
    oracle on every row and on the stored 1/rms: ordinary rows; a gamma with
    one huge entry (2^31) on a column that is zero in every row, which
    changes no Xn; and zero rows and constant rows mixed in."""
    T, K = 2048, 4096          # 2048 one-row CTAs do not fit at once: the wide form
    x = synthetic.activations(811, T, K)
    gamma = synthetic.gamma(812, K)
    if case == "huge_gamma_on_zero_column":
        x[:, 17] = 0.0
        gamma[17] = np.float32(2.0 ** 31)
    elif case == "mixed":
        x[::7] = 0.0                                  # zero rows: P = 0
        x[3::7] = np.float32(0.75)                    # constant rows: every product equal up to gamma
        gamma[::2] = np.float32(1.0)
    act = _gpu_prep(x, gamma, 1e-5)
    got = _read(act, T, K, sq.SHARQ_MODE_SHARQ)
    p = O.prep(x, gamma, 1e-5)
    assert got["s_g"] == float(p["s_g"])
    for f in ("meta", "sp_codes", "sp_sf", "r_codes", "r_sf"):
        _assert_equal(f, got[f][:T], p[f])
    inv = act.region("inv_rms", 4 * T).view(torch.float32).cpu().numpy()
    assert np.array_equal(inv.view(np.uint32), p["inv"].view(np.uint32))
