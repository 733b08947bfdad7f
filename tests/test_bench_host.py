"""Host-side bench logic (CPU): the algorithmic byte counts behind the
roofline fractions, the workload shapes, and the kernel the report names.

Prep: 2 B read and 0.90625 B written per activation element (bf16 in;
backbone codes 0.25 + scales 1/32, metadata 1/16, residual codes 0.5 +
scales 1/16).  GEMM: the packed weight (0.5 codes + 1/16 + 1/32 scales =
0.59375 B per weight), the prepared activation of the 128-padded rows and
the bf16 output.
"""
import pytest

import bench


def test_prep_bytes_per_element():
    # the output formats, byte by byte per activation element
    out = 0.25 + 1 / 32 + 1 / 16 + 0.5 + 1 / 16
    assert out == 0.90625
    assert bench.prep_alg_bytes(8192, 18944) == 8192 * 18944 * (2 + out)
    # padding rows are not touched: T = 1 moves one row
    assert bench.prep_alg_bytes(1, 4096) == 4096 * (2 + out)


def test_gemm_bytes_q_proj_decode():
    w = 0.5 + 1 / 16 + 1 / 32
    assert w == 0.59375
    b = bench.gemm_alg_bytes(1, 4096, 4096)
    assert b == 4096 * 4096 * w + 128 * 4096 * 0.90625 + 4096 * 2
    assert 10.4e6 < b < 10.5e6          # ~1.6 us at 6.55 TB/s


def test_qwen_layer_workload_shapes_and_flops():
    layers = bench.workload_layers("qwen_layer", [1, 64, 1024, 8192])
    assert len(layers) == 16
    shapes = {(L.K, L.D, L.norm) for L in layers}
    assert shapes == {(3584, 4608, True), (3584, 3584, False), (3584, 37888, True), (18944, 3584, False)}
    assert sum(L.flops for L in layers if L.T == 8192) == pytest.approx(
        2 * 8192 * (3584 * 4608 + 3584 * 3584 + 3584 * 37888 + 18944 * 3584))


@pytest.mark.parametrize("T,K,D,name", [
    (8192, 3584, 37888, "sharq_gemm_pair_kernel"),      # prefill: CTA pairs
    (1, 3584, 4608, "sharq_gemm_kernel (split-K)"),     # 18 column tiles: split-K
    (1, 3584, 37888, "sharq_gemm_persistent_kernel"),   # one row tile, 148 column tiles
])
def test_kernel_named_in_the_report(T, K, D, name):
    L = bench.Layer("x", T, K, D, False)
    assert bench.gemm_kernel_name(L) == name
