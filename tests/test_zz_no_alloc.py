"""sharq_prep_noalloc: the allocation-free prep entry point (GPU).

For callers that cannot allocate device memory (runtimes whose memory
planner owns the GPU, serving loops that must not call cudaMalloc),
sharq_prep_noalloc keeps the prep's working memory in a fixed array inside
the library.  Called through
the C ABI, it must give exactly sharq_prep's outputs -- and the oracle's, bit
for bit on every row -- and keep doing so on the next call (the array keeps
the previous call's contents).  The cases cover the single-launch form and the
wide two-launch form, which keeps each row's 1/rms in the array.  This file
is collected last so that a failure here comes after every other test has run.
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


def _outputs(act, T, K):
    Tp = act.view.Tp
    tiles = (Tp // 128) * (K // 256)
    out = {}
    for name, per_tile in (("r_codes", 16384), ("r_sf", 2048), ("sp_codes", 8192), ("meta", 2048),
                           ("sp_sf", 1024)):
        rows = act.region(name, tiles * per_tile).cpu().numpy().reshape(Tp // 128, K // 256, 128, -1)
        out[name] = rows  # compared whole tiles; rows >= T are untouched by both calls
    out["s_g"] = act.region("s_g", 4).view(torch.float32).item()
    return out


def _check_oracle(out, x, gamma, T, K):
    """every row of the prepared operands against the oracle, bit for bit"""
    p = O.prep(x, gamma, 1e-5)
    assert out["s_g"] == float(p["s_g"])
    Tp = -(-T // 128) * 128
    flat = lambda name: out[name].reshape(-1)
    assert np.array_equal(_layout.untile_meta(flat("meta"), Tp, K)[:T], p["meta"])
    assert np.array_equal(_layout.untile_sp_codes(flat("sp_codes"), Tp, K)[:T], p["sp_codes"])
    assert np.array_equal(_layout.untile_sf(flat("sp_sf"), Tp, K, 32)[:T], p["sp_sf"])
    assert np.array_equal(_layout.untile_codes(flat("r_codes"), Tp, K)[:T], p["r_codes"])
    assert np.array_equal(_layout.untile_sf(flat("r_sf"), Tp, K, 16)[:T], p["r_sf"])


# (16, 4096): one thread-block cluster; (300, 1024): the grid-barrier form;
# (400, 14336): the wide two-launch form (per-row 1/rms kept in the array)
@pytest.mark.parametrize("T,K,D", [(16, 4096, 1024), (300, 1024, 512), (400, 14336, 256)])
def test_noalloc_prep_matches_prep_on_consecutive_calls(T, K, D):
    stream = torch.cuda.current_stream().cuda_stream
    gamma = H.bf16_dev(synthetic.gamma(5, K))
    pw = sq.PackedWeight(torch.from_numpy(synthetic.weights(6, K, D)).to(torch.bfloat16).cuda())
    for call, seed in enumerate((11, 12)):      # two calls in a row, different inputs
        xh = synthetic.activations(seed, T, K)
        x = H.bf16_dev(xh)
        ref = sq.PreparedAct(T, K)
        ref.buf.zero_()
        ref.prep(x, gamma, 1e-5)
        got = sq.PreparedAct(T, K)
        got.buf.zero_()
        sq.sharq_prep_noalloc(x.data_ptr(), gamma.data_ptr(), 1e-5, None, got.view, stream)
        torch.cuda.synchronize()
        a, b = _outputs(ref, T, K), _outputs(got, T, K)
        assert a["s_g"] == b["s_g"], call
        for name in ("r_codes", "r_sf", "sp_codes", "meta", "sp_sf"):
            assert np.array_equal(a[name], b[name]), (call, name)
        _check_oracle(b, xh, synthetic.gamma(5, K), T, K)
        ya = sq.linear(ref, pw, out_dtype=torch.float32)
        yb = sq.linear(got, pw, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(ya, yb), call


def test_noalloc_rejects_too_many_rows():
    act = sq.sharq_act_view(1 << 20, 16385, 256)   # view only; rejected before any device work
    with pytest.raises(sq.SharqError) as e:
        sq.sharq_prep_noalloc(1 << 22, None, 1e-5, None, act, None)
    assert e.value.status == -2
