"""moe_combine and moe_load_stats through their own entry points.

The layer runs both inside one launch (the combine kernel plus its
statistics CTA); these tests call the standalone entry points, which take
their inputs from the caller, and compare them with the oracle's combine
and load statistics on the same inputs.
"""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O
from tests.gpu_util import dev, f64

pytestmark = pytest.mark.gpu


def _combine_inputs(T, K, d, drop, seed):
    """inv [T, K] (distinct rows 0..N-1, or -1 with probability `drop`; every
    7th token fully dropped), weights w [T, K] fp32, Y_perm [N + 8, d] fp32
    whose last 8 rows (never referenced) are NaN."""
    rng = np.random.default_rng(seed)
    kept = rng.random((T, K)) >= drop
    kept[::7] = False
    N = int(kept.sum())
    rows = rng.permutation(N)
    inv = np.full((T, K), -1, np.int32)
    inv[kept] = rows
    w = np.abs(synth.normal_f32(T * K, seed, synth.STREAM_MISC).numpy()).reshape(T, K).astype(np.float32)
    Y = synth.normal_f32((N + 8) * d, seed, synth.STREAM_LOGITS).reshape(N + 8, d) * 3.0
    Y[N:] = float("nan")
    return inv, w, Y.to(torch.float32), N


@pytest.mark.parametrize("T,K,d,drop", [(1, 1, 16, 0.0), (300, 2, 4096, 0.0), (257, 8, 7168, 0.3),
                                        (1000, 4, 2048, 0.5), (64, 16, 128, 0.1)])
def test_combine_matches_oracle(T, K, d, drop):
    inv, w, Y, N = _combine_inputs(T, K, d, drop, seed=T + K)
    dims = abi.Dims(T, d, 64, max(K, 8), K)
    y = torch.full((T, d), float("nan"), dtype=torch.float32, device=dev())
    abi.moe_combine(dims, Y.to(dev()), torch.from_numpy(inv).to(dev()), torch.from_numpy(w).to(dev()), y)
    torch.cuda.synchronize()
    Y64 = Y.double().numpy()
    ref = O.combine(Y64, inv, w.astype(np.float64), T)
    yg = f64(y)
    assert np.all(np.isfinite(yg))  # the NaN rows are never read
    # fp32 fused multiply-adds in slot order: |error| <= gamma_K * sum_k |w_k Y_k|
    absum = np.zeros((T, d))
    for k in range(K):
        r = inv[:, k]
        live = r >= 0
        absum[live] += np.abs(w[live, k].astype(np.float64))[:, None] * np.abs(Y64[r[live]])
    u = 2.0 ** -24
    gamma = K * u / (1 - K * u)
    assert np.all(np.abs(yg - ref) <= gamma * absum + 1e-30)
    dead = np.all(inv < 0, axis=1)
    assert dead.any() and np.all(yg[dead] == 0.0)


@pytest.mark.parametrize("T,E,K,with_P", [(256, 8, 2, True), (4096, 256, 8, True), (8192, 60, 4, False),
                                          (1, 1, 1, True)])
def test_load_stats_matches_oracle(T, E, K, with_P):
    idx = synth.distinct_choices(T, E, K, seed=T + E).numpy()
    counts = O.expert_counts(idx, E).astype(np.int32)
    P = np.abs(synth.normal_f32(E, E, synth.STREAM_MISC).numpy()).astype(np.float32) + 0.01
    P = (P / P.sum()).astype(np.float32)
    dims = abi.Dims(T, 128, 256, E, K)
    f = torch.full((E,), float("nan"), dtype=torch.float32, device=dev())
    aux = torch.full((1,), float("nan"), dtype=torch.float32, device=dev())
    Pd = torch.from_numpy(P).to(dev()) if with_P else None
    abi.moe_load_stats(dims, torch.from_numpy(counts).to(dev()), Pd, f, aux if with_P else None)
    torch.cuda.synchronize()
    f_o, P_o, aux_o = O.load_stats(counts, np.repeat(P.astype(np.float64)[None, :], T, axis=0), T, K)
    fg = f64(f)
    # fp32 count * fp32(1 / (T K)): two roundings
    assert np.all(np.abs(fg - f_o) <= 2 * 2.0 ** -24 * f_o + 1e-30)
    assert abs(fg.sum() - 1.0) <= 1e-5
    if with_P:
        assert np.allclose(P_o, P.astype(np.float64), rtol=1e-12, atol=0)
        assert abs(float(aux.item()) - aux_o) <= 1e-5 * max(1.0, aux_o)
    else:
        assert np.isnan(float(aux.item()))  # not written


def test_combine_bf16_output_is_rne_of_fp32():
    T, K, d = 513, 4, 1024
    inv, w, Y, N = _combine_inputs(T, K, d, 0.2, seed=11)
    dims = abi.Dims(T, d, 64, 8, K)
    args = (Y.to(dev()), torch.from_numpy(inv).to(dev()), torch.from_numpy(w).to(dev()))
    y32 = torch.empty(T, d, dtype=torch.float32, device=dev())
    y16 = torch.empty(T, d, dtype=torch.bfloat16, device=dev())
    abi.moe_combine(dims, *args, y32)
    abi.moe_combine(dims, *args, y16)
    torch.cuda.synchronize()
    assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
