"""sharq_prep_linear: the fused single-kernel decode form (GPU).

For T <= 32 the GEMM CTAs prepare the activation themselves; the result must
equal sharq_prep + sharq_linear exactly (same codes, same MMA order), and
match the oracle.  Above 32 rows the call runs the two kernels.
"""
import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
import synthetic
from oracle import sharq as O
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


@pytest.mark.parametrize("T,K,D,norm", [
    (1, 4096, 4096, True), (5, 4096, 4096, True), (16, 4096, 4096, True), (32, 768, 384, False),
    (7, 256, 256, True), (3, 18944, 3584, False), (2, 3584, 37888, True), (33, 1024, 512, True)])
def test_fused_equals_two_kernels_and_oracle(T, K, D, norm):
    x = synthetic.activations(600 + T, T, K)
    gamma = synthetic.gamma(601, K) if norm else None
    w = synthetic.weights(602, K, D)
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    xd = H.bf16_dev(x)
    gd = H.bf16_dev(gamma) if norm else None
    for dt in (torch.float32, torch.bfloat16):
        y_fused = sq.prep_linear(xd, gd, 1e-5, pw, out_dtype=dt)
        act = sq.PreparedAct(T, K)
        act.prep(xd, gd, 1e-5)
        y_two = sq.linear(act, pw, out_dtype=dt)
        torch.cuda.synchronize()
        assert torch.equal(y_fused, y_two), (dt, (y_fused.float() - y_two.float()).abs().max().item())
    ref = O.linear(O.prep(x, gamma, 1e-5), O.pack_weight(w))
    y = sq.prep_linear(xd, gd, 1e-5, pw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert H.rel_fro(y.cpu().numpy(), ref) < 1e-5


def test_fused_consecutive_calls_and_empty():
    K, D = 4096, 1024
    w = synthetic.weights(610, K, D)
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    gd = H.bf16_dev(synthetic.gamma(611, K))
    for seed in (1, 2, 3):
        x = synthetic.activations(620 + seed, 4, K)
        y = sq.prep_linear(H.bf16_dev(x), gd, 1e-5, pw, out_dtype=torch.float32)
        torch.cuda.synchronize()
        ref = O.linear(O.prep(x, synthetic.gamma(611, K), 1e-5), O.pack_weight(w))
        assert H.rel_fro(y.cpu().numpy(), ref) < 1e-5
    y0 = sq.prep_linear(torch.empty((0, K), dtype=torch.bfloat16, device="cuda"), gd, 1e-5, pw)
    assert y0.shape == (0, D)
