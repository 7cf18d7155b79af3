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


def test_router_bytes_are_features_and_weights_once():
    w = W.WORKLOADS["flash_2b_13tiles"]
    x = T * 1024 * C * 2
    pool_w = 2 * 4 * 4 * D * D        # Wq, Wk, Wv, Wo of 4 layers, bf16
    gate_w = 2 * 4 * 2 * D * 1024     # W1 and W2 of 4 gating blocks, bf16
    b = bench.router_bytes(w, T)
    assert x + pool_w + gate_w < b < (x + pool_w + gate_w) * 1.01
    assert abs(b - 77.7e6) < 0.2e6    # 27.3 MB of features + 33.5 + 16.8 MB of weights


def test_clock_summary_separates_the_timed_window():
    lines = [
        "2026/12/03 10:00:00.000, 0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/03 10:00:00.500, 0, 1950, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/03 10:00:01.000, 0, 1965, 1965, 650.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    rows = bench.ClockSampler.parse(lines)
    assert len(rows) == 3
    t0, t1 = rows[0][0], rows[2][0]
    s = bench.ClockSampler.summarise(rows, t0, t1)
    assert s["samples"] == 3 and s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 900.0
    assert bench.ClockSampler.summarise(rows, t1 + 10, t1 + 20)["reasons"] == ["unsampled"]


def test_cpu_sample_plans():
    """Whole images (routing couples an image's tiles) on the flash
    workloads, 8 seeded tiles of the large connector batches."""
    import torch
    w2 = W.WORKLOADS["flash_2b_13tiles"]
    inp = {"workload": w2, "T": 13, "image_offsets": torch.tensor([0, 13], dtype=torch.int32)}
    assert bench.cpu_sample_plan(inp) == ("images", 1)
    w3 = W.WORKLOADS["flash_4b_batched"]
    offs = torch.tensor([0, 3, 5, 12, 20, 31, 40, 41, 50, 60, 70, 80, 90, 97, 100, 105, 110],
                        dtype=torch.int32)
    kind, n = bench.cpu_sample_plan({"workload": w3, "T": 110, "image_offsets": offs})
    assert kind == "images" and offs[n] >= 8 and offs[n - 1] < 8
    w4 = W.WORKLOADS["connector_14b_832tiles"]
    kind, tiles = bench.cpu_sample_plan({"workload": w4, "T": 832})
    assert kind == "tiles" and len(tiles) == 8 and len(set(tiles)) == 8 and max(tiles) < 832
