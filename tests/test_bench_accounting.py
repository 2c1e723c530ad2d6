"""The bench's roofline accounting (host only): algorithmic bytes and FLOPs."""
import numpy as np

import bench
from moe_layer_gemm_b200 import synth


def test_decode_layer_bytes_and_flops():
    wl = synth.get_workload("mixtral_decode")
    counts = np.array([64] * 8)
    alg = bench.layer_algorithmic(wl, counts, counts)
    d, f, T, E, K = 4096, 14336, 256, 8, 2
    weights = E * 3 * d * f * 2                       # every expert touched, bf16
    assert alg["touched"] == E and alg["n_kept"] == T * K
    assert alg["layer_bytes"] == weights + T * d * 2 + T * d * 4 + d * E * 2
    assert alg["layer_flops"] == 2 * T * d * E + 6 * d * f * T * K
    assert alg["gemm_bytes"] == weights           # touched expert weights only
    assert alg["gemm_design_bytes"] == T * K * (d * 2 + 2 * f * 2 + d * 4)
    assert alg["gemm_flops"] == 6 * d * f * T * K
    # the decode layer is HBM-bound at the measured peaks: 2.8 GB vs 180 GFLOP
    assert alg["layer_bytes"] / 6541e9 > alg["layer_flops"] / 1627e12


def test_untouched_and_dropped_experts_are_not_counted():
    wl = synth.get_workload("qwen_capacity")
    counts = np.zeros(wl.E, dtype=np.int64)
    counts[:3] = [900, 10, 547]
    kept = np.minimum(counts, 547)
    alg = bench.layer_algorithmic(wl, counts, kept)
    assert alg["touched"] == 3
    assert alg["n_kept"] == 547 + 10 + 547
    assert alg["gemm_flops"] == 6 * wl.d_model * wl.d_ff * alg["n_kept"]
