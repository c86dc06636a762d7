"""Host-side checks of the figures bench.py reports (no GPU).

The roofline line divides algorithmic bytes or flops by a measured time, and
`gpu_launches` claims how many library kernels one step runs; both come from
small pure-Python functions that are checked here against hand counts.
"""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_rl_fine_b200 import accounting as A  # noqa: E402
from quantized_rl_fine_b200 import configs as C  # noqa: E402


def test_bytes_per_parameter_of_the_two_bases():
    # 4-bit codes plus one scale per 32 elements: BF16 (INT4) or E8M0 (MXFP4)
    assert A.bytes_per_param("int4") == 0.5 + 2 / 32
    assert A.bytes_per_param("mxfp4") == 0.5 + 1 / 32
    N, K = 4096, 7168
    assert A.expert_weight_bytes(N, K, "int4") == N * K // 2 + N * (K // 32) * 2
    assert A.expert_weight_bytes(N, K, "int4") == int(A.bytes_per_param("int4") * N * K)
    assert A.expert_weight_bytes(N, K, "mxfp4") == int(A.bytes_per_param("mxfp4") * N * K)


def test_flops_and_weight_bytes_count_only_real_rows_and_active_experts():
    rows = [3, 0, 5, 0, 1]
    N, K = 256, 512
    assert A.gemm_flops(rows, N, K) == 2 * 9 * N * K
    assert A.active_weight_bytes(rows, N, K, "mxfp4") == 3 * A.expert_weight_bytes(N, K, "mxfp4")
    assert A.active_weight_bytes([0, 0], N, K, "int4") == 0


def test_step_accounting_of_an_up_projection():
    cfg = C.MXFP4_UP
    counts = [64] * cfg.E
    acc = bench._accounting(cfg, counts)
    M = sum(counts)
    assert acc["flops"] == 2 * M * cfg.f * cfg.d
    wb = cfg.E * A.expert_weight_bytes(cfg.f, cfg.d, "mxfp4")
    assert acc["wbytes"] == wb
    # weights once, the permuted input rows and the output rows
    assert acc["gemm"]["bytes"] == wb + M * cfg.d * 2 + M * cfg.f * 2


def test_step_accounting_of_a_training_step_with_adapter():
    cfg = C.TINY_INT4.with_(adapter=True, train=True)
    counts = [5, 0, 7, 4, 0, 0, 3, 5]
    acc = bench._accounting(cfg, counts)
    M = sum(counts)
    d, f = cfg.d, cfg.f
    gu, dn = 2 * M * (2 * f) * d, 2 * M * d * f
    # forward and backward GEMMs, adapter forward (2 M d 32) and backward (4 M d 32)
    assert acc["flops"] == 2 * (gu + dn) + 2 * M * d * 32 + 4 * M * d * 32
    active = sum(1 for c in counts if c)
    assert acc["wbytes"] == 2 * active * (A.expert_weight_bytes(2 * f, d, "int4")
                                          + A.expert_weight_bytes(d, f, "int4"))


@pytest.mark.parametrize("cfg,kernels", [
    # top-k, routing tail (offsets, permutation, row copy), up GEMM
    (C.MXFP4_UP, 3),
    # top-k, tail, gate/up, down, combine
    (C.TRILLION_INT4.with_(T=128), 5),
    # top-k, scan, scatter, row copy, gate/up, down, combine
    (C.TRILLION_INT4.with_(T=2048), 7),
    # routing (3), adapter (gathers the rows), gate/up, down, combine, scatter
    # of dy, two backward GEMMs, fused adapter backward, combine of dx
    (C.TRAIN_INT4, 12),
    # top-k, scan, scatter, row copy, gate/up and down as two launches each
    # (narrow and wide experts: 341 rows per expert on average), combine
    (C.TRILLION_INT4.with_(T=16384), 9),
    # the same for the Zipf-routed MXFP4 layer (256 rows per expert on average)
    (C.ZIPF_MXFP4, 9),
])
def test_launch_count_per_step(cfg, kernels):
    assert bench._launches_per_step(cfg) == kernels
