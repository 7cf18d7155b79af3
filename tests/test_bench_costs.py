"""The algorithmic costs bench.py divides by kernel time (the roofline
numerators) against the layer shapes written out by hand (runs without a GPU).

Shapes of the 13-tile InternVL3.5-2B-Flash workload: C = 1024 ViT channels,
H = 2048 LLM width, mlp2 intermediate 4096; pixel_shuffle at 0.5 gives 256 rows
of 4C per tile, at 0.25 64 rows of 16C; 1024 tokens per tile, D = 1024."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402

T = 13
C, H, MID, D = 1024, 2048, 4096, 1024


def _alg():
    w = W.WORKLOADS["flash_2b_13tiles"]
    assert (w.C, w.H, w.mlp2_mid, w.D) == (C, H, MID, D)
    return bench.algorithmic(w, T)


def test_connector_gemm_flops_are_two_m_n_k():
    alg = _alg()
    shapes = {  # rows, K, N of each Linear for the whole image
        "mlp1.fc1": (T * 256, 4 * C, H),
        "mlp1.fc2": (T * 256, H, H),
        "mlp2.fc1": (T * 64, 16 * C, MID),
        "mlp2.fc2": (T * 64, MID, H),
        "mlp2.fc3": (T * 64, H, H),
    }
    for role, (m, k, n) in shapes.items():
        assert alg[role][0] == 2 * m * k * n, role


def test_dominant_kernel_bytes_are_x_weights_and_output_once():
    alg = _alg()
    x = T * 1024 * C * 2            # the features, read through the 5-D TMA view
    w0 = 16 * C * MID * 2           # the folded first Linear of mlp2
    y = T * 64 * MID * 2            # its bf16 output
    assert alg["mlp2.fc1"][1] == x + w0 + y
    assert abs(alg["mlp2.fc1"][1] - 168.3e6) < 0.1e6


def test_single_pass_attention_counts_both_contractions_and_one_read_of_x():
    alg = _alg()
    assert alg["pool.attend"][0] == alg["pool.scores"][0] + alg["pool.wsum"][0]
    x_per_layer = T * 1024 * D * 2
    # four layers, each reading x once (the tensor-core form reads it twice)
    assert 4 * x_per_layer < alg["pool.attend"][1] < 4 * x_per_layer * 1.1
    assert alg["pool.scores"][1] + alg["pool.wsum"][1] > 8 * x_per_layer
