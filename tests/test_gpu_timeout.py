"""A device-side bounded wait that runs out (GPU).

The single-launch prep of a tensor that needs more CTAs than one cluster holds
meets at a grid barrier for the per-tensor max.  The test names one CTA in
the act's fault-injection word, so that CTA never arrives and every CTA's
bounded wait (2 s) runs out.  No fault, trap or endless loop is involved: the
kernel records SHARQ_ERR_TIMEOUT, sharq_linear forwards it to its workspace,
sharq_check_status returns it, and the next call on the same buffers (word
cleared) is clean and bit-exact.
"""
import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
import synthetic
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
SHARQ_ERR_TIMEOUT = -5


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def test_grid_barrier_timeout_is_reported_and_cleared():
    T, K, D = 128, 4096, 256          # 128 CTAs of one row each: the grid-barrier form
    x = H.bf16_dev(synthetic.activations(71, T, K))
    gamma = H.bf16_dev(synthetic.gamma(72, K))
    pw = sq.PackedWeight(torch.from_numpy(synthetic.weights(73, K, D)).to(torch.bfloat16).cuda())
    ws = sq.Workspace(T, K, D)
    act = sq.PreparedAct(T, K)
    words = act.region("gmax_bits", 24).view(torch.int32)

    words[5] = 1                      # CTA 0 skips its arrival
    act.prep(x, gamma, 1e-5)
    sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    assert ws.check() == SHARQ_ERR_TIMEOUT
    w = words.cpu().numpy()
    assert w[3] == SHARQ_ERR_TIMEOUT  # the prep's error word
    assert w[0] == 0 and w[1] == 0 and w[2] == 0 and w[4] == 0   # counters reset by the last CTA out

    words[5] = 0
    act.prep(x, gamma, 1e-5)
    y = sq.linear(act, pw, out_dtype=torch.float32, ws=ws)
    assert ws.check() == 0
    assert words.cpu().numpy()[3] == 0
    ref = sq.PreparedAct(T, K)
    ref.prep(x, gamma, 1e-5)
    ws2 = sq.Workspace(T, K, D)
    y_ref = sq.linear(ref, pw, out_dtype=torch.float32, ws=ws2)
    assert ws2.check() == 0
    assert torch.equal(y, y_ref)
    n = act.view.r_sf - act.view.r_codes
    assert torch.equal(act.region("r_codes", n), ref.region("r_codes", n))
