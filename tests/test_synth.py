"""The seeded input generator: determinism, slicing, distribution."""
import numpy as np
import torch

from moe_layer_gemm_b200 import synth


def test_known_hash_values():
    # lowbias32 reference values (the published hash, computed with Python ints)
    x = torch.tensor([0, 1, 2, 0xFFFFFFFF], dtype=torch.int64)
    got = synth._lowbias32(x).tolist()
    assert got == [synth._lowbias32_int(int(v)) for v in x]
    # and against an independent uint64 numpy evaluation
    v = np.array([0, 1, 2, 0xFFFFFFFF], dtype=np.uint64)
    m = np.uint64(0xFFFFFFFF)
    v ^= v >> np.uint64(16); v = (v * np.uint64(0x7FEB352D)) & m
    v ^= v >> np.uint64(15); v = (v * np.uint64(0x846CA68B)) & m
    v ^= v >> np.uint64(16)
    assert got == v.tolist()


def test_chunking_and_offsets_do_not_change_values():
    a = synth.normal_bf16((37, 41), seed=5, stream=synth.STREAM_X, chunk=1 << 20)
    b = synth.normal_bf16((37, 41), seed=5, stream=synth.STREAM_X, chunk=100)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    tail = synth.normal_f32(50, 5, synth.STREAM_X, offset=37 * 41 - 50)
    assert torch.equal(tail.to(torch.bfloat16).view(torch.int16), a.reshape(-1)[-50:].view(torch.int16))


def test_offsets_past_2_pow_32():
    n0 = (1 << 32) - 3
    a = synth.normal_f32(6, 1, synth.STREAM_W1, offset=n0)
    b = torch.cat([synth.normal_f32(3, 1, synth.STREAM_W1, offset=n0),
                   synth.normal_f32(3, 1, synth.STREAM_W1, offset=n0 + 3)])
    assert torch.equal(a, b)


def test_expert_slabs_equal_full_tensor_slices():
    wl = synth.get_workload("tiny")
    W1, W3, W2 = synth.make_expert_weights(wl)
    s1, s3, s2 = synth.make_expert_weights(wl, experts=[5, 2])
    for full, part in ((W1, s1), (W3, s3), (W2, s2)):
        assert torch.equal(full[[5, 2]].view(torch.int16), part.view(torch.int16))


def test_streams_and_seeds_differ():
    a = synth.normal_f32(1000, 0, synth.STREAM_X)
    b = synth.normal_f32(1000, 0, synth.STREAM_WR)
    c = synth.normal_f32(1000, 1, synth.STREAM_X)
    assert not torch.equal(a, b) and not torch.equal(a, c)


def test_normal_moments():
    v = synth.normal_f32(1 << 20, 3, synth.STREAM_X).double()
    assert abs(v.mean().item()) < 5e-3
    assert abs(v.var().item() - 1) < 1e-2
    k = ((v - v.mean()) ** 4).mean() / v.var() ** 2
    assert abs(k.item() - 3) < 0.05


def test_distinct_choices_rows_are_distinct():
    idx = synth.distinct_choices(200, 12, 5, seed=3)
    assert idx.shape == (200, 5) and idx.dtype == torch.int32
    for row in idx.tolist():
        assert len(set(row)) == 5 and all(0 <= e < 12 for e in row)


def test_tie_logits_have_ties_and_signed_zeros():
    l = synth.logits_f32(400, 8, seed=2, tie_frac=0.5)
    zeros = l == 0
    assert zeros.any()
    assert (torch.signbit(l) & zeros).any() and (~torch.signbit(l) & zeros).any()


def test_workload_calibration_loaded():
    w = synth.workloads()
    assert len(w["mixtral_prefill"].skew_params["scales"]) == 8
    assert len(w["qwen_capacity"].skew_params["hot"]) == 6
    assert len(w["deepseek_bias"].skew_params["scales"]) == 256
