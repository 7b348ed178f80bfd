"""The algorithmic work bench.py divides by (the roofline numerators), counted independently from the
seeded weights' shapes, and the DM0-base figures they must give: 15.73 M action-expert and 50.33 M VLM
parameters per layer (matrices only), 974.4 MB of HBM per single-observation Euler step (bf16
weights plus the 816-token prefix cache read once), 1.649 TFLOP per batched gate/up launch."""
import numpy as np
import pytest

import bench
from synth import inputs as I

D = I.DM0_BASE


@pytest.mark.parametrize("branch", [0, 1])
def test_layer_params_counts_the_weight_matrices(branch):
    shapes = I.layer_shapes(D, branch)
    matrices = sum(int(np.prod(s)) for n, s in shapes.items() if len(s) == 2)
    assert bench.layer_params(D, branch) == matrices
    assert matrices == (50_331_648 if branch == 0 else 15_728_640)


def test_denoise_bytes_per_euler_step():
    weights = D.layers * 15_728_640 * 2
    kv = D.layers * 1 * D.n_kv * 816 * D.head_dim * 2 * 2
    assert (weights, kv) == (880_803_840, 93_585_408)
    assert bench.denoise_bytes_per_step(D, 1, 816) == weights + kv == 974_389_248


def test_gate_up_flops_of_the_batched_prefix_pass():
    assert bench.prefill_gateup_flops(D, 16, 2048) == 2 * 16 * 2048 * 2048 * 2 * 6144
    assert abs(bench.prefill_gateup_flops(D, 16, 2048) / 1e12 - 1.649) < 1e-3


def test_merged_layer_flops():
    # one DM0-base layer over 816 prefix + 50 suffix tokens: 83.7 GFLOP of GEMM (82.1 VLM + 1.6 action)
    # and 5.8 GFLOP of attention (prefix rows over 816 keys, suffix rows over 866, QK^T and PV)
    gemm, attn = bench.merged_layer_flops(D, 816, 50)
    assert gemm == 2 * 816 * 50_331_648 + 2 * 50 * 15_728_640
    assert round(gemm / 1e9, 1) == 83.7 and round(attn / 1e9, 1) == 5.8
