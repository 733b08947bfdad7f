"""The CTA-pair prefill GEMM (tcgen05 cta_group::2, 256 x 256 tiles) (GPU).

sharq_linear runs ungrouped SharQ and plain-NVFP4 GEMMs with at least two
128-row tiles whose output tiles fill the GPU on CTA pairs.  These cases pin
it against the oracle where its own logic could go wrong: an odd number of
128-row tiles (the last pair's second CTA lies past the activation's end and
copies no activation bytes), a ragged last tile, both operand sets, both
output types and the per-token scale mode; and against the one-CTA persistent
kernel on the same shapes (SHARQ_GEMM_PAIR=0 in a child process).
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import sparse_activation_quantization_b200 as sq
import synthetic
from oracle import sharq as O
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# 3 row tiles (T = 300: ragged, odd) x 25 column tiles of 256: 75 output
# tiles, enough that sharq_linear takes the persistent (not split-K) route
T, K, D = 300, 1024, 6400


@pytest.fixture(scope="module", autouse=True)
def _built():
    H.ensure_built()


def _inputs():
    x = synthetic.activations(61, T, K)
    gamma = synthetic.gamma(62, K)
    w = synthetic.weights(63, K, D)
    return x, gamma, w


def _gpu(x, gamma, w, mode, out_dtype):
    pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
    act = sq.PreparedAct(T, K, mode)
    act.prep(H.bf16_dev(x), H.bf16_dev(gamma), 1e-5)
    ws = sq.Workspace(T, K, D)
    y = sq.linear(act, pw, out_dtype=out_dtype, ws=ws)
    torch.cuda.synchronize()
    assert ws.check() == 0
    return y.float().cpu().numpy()


@pytest.mark.parametrize("mode", [sq.SHARQ_MODE_SHARQ, sq.SHARQ_MODE_NVFP4, sq.SHARQ_MODE_SHARQ_TOKEN],
                         ids=["sharq", "nvfp4", "sharq_per_token"])
def test_pair_gemm_matches_oracle(mode):
    x, gamma, w = _inputs()
    q = O.pack_weight(w)
    if mode == sq.SHARQ_MODE_NVFP4:
        ref = O.linear_nvfp4(O.prep_nvfp4(x, gamma, 1e-5), q)
    elif mode == sq.SHARQ_MODE_SHARQ_TOKEN:
        ref = O.linear(O.prep_per_token(x, gamma, 1e-5), q)
    else:
        ref = O.linear(O.prep(x, gamma, 1e-5), q)
    y32 = _gpu(x, gamma, w, mode, torch.float32)
    # every (128-row, 256-column) output tile, the ragged and odd ones included
    for lo in range(0, T, 128):
        for c in range(0, D, 256):
            e = H.rel_fro(y32[lo:lo + 128, c:c + 256], ref[lo:lo + 128, c:c + 256])
            assert e < 1e-5, (lo, c, e)
    yb = _gpu(x, gamma, w, mode, torch.bfloat16)
    assert H.rel_fro(yb, ref) <= 1e-3 + 2.0 ** -8
    assert np.all(np.abs(yb - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max())


_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import sparse_activation_quantization_b200 as sq, synthetic
T, K, D = int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4])
x = synthetic.activations(61, T, K); g = synthetic.gamma(62, K); w = synthetic.weights(63, K, D)
pw = sq.PackedWeight(torch.from_numpy(w).to(torch.bfloat16).cuda())
act = sq.PreparedAct(T, K)
act.prep(torch.from_numpy(x).to(torch.bfloat16).cuda(), torch.from_numpy(g).to(torch.bfloat16).cuda(), 1e-5)
y = sq.linear(act, pw, out_dtype=torch.float32)
torch.cuda.synchronize()
np.save(sys.argv[5], y.cpu().numpy())
"""


def test_pair_and_single_cta_forms_agree(tmp_path):
    x, gamma, w = _inputs()
    y_pair = _gpu(x, gamma, w, sq.SHARQ_MODE_SHARQ, torch.float32)
    out = tmp_path / "y_single.npy"
    env = dict(os.environ, SHARQ_GEMM_PAIR="0")
    subprocess.run([sys.executable, "-c", _CHILD, ROOT, str(T), str(K), str(D), str(out)], env=env, check=True,
                   timeout=600)
    y_single = np.load(out)
    assert H.rel_fro(y_pair, y_single) < 1e-6
