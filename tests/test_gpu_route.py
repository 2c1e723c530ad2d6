"""Router parity: top-K, renormalisation, P_i (bit-exact selection on shared logits)."""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O
from tests.gpu_util import (P_TOL, W_TOL, ambiguous_tokens, check_routing_validity, dev, f64)

pytestmark = pytest.mark.gpu


def _bias(E, seed, scale=0.5):
    return (synth.normal_f32(E, seed, synth.STREAM_MISC) * scale).to(torch.float32)


@pytest.mark.parametrize("T,E,K,use_bias,tie", [
    (1000, 8, 2, False, 0.3), (777, 60, 4, True, 0.3), (513, 256, 8, True, 0.3), (64, 1, 1, False, 0.0),
    (100, 16, 16, False, 0.5), (300, 33, 5, True, 0.2), (1, 8, 2, False, 0.0), (4097, 128, 6, True, 0.1)])
def test_route_from_logits_bitexact(T, E, K, use_bias, tie):
    d = dev()
    logits = synth.logits_f32(T, E, seed=T + E, tie_frac=tie, device=d)
    bias = _bias(E, T).to(d) if use_bias else None
    dims = abi.Dims(T, 128, 256, E, K)
    ws = abi.alloc_workspace(dims)
    idx = torch.empty(T, K, dtype=torch.int32, device=d)
    w = torch.empty(T, K, dtype=torch.float32, device=d)
    P = torch.empty(E, dtype=torch.float32, device=d)
    abi.moe_route_from_logits(dims, logits, bias, idx, w, P, ws)
    torch.cuda.synchronize()
    l_host = logits.cpu().numpy()
    b_host = None if bias is None else bias.cpu().numpy()
    idx_o, w_o, _ = O.route_from_logits_f32(l_host, K, b_host)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.max(np.abs(f64(w) - w_o)) <= W_TOL
    P_o = O.softmax_rows(l_host.astype(np.float64)).mean(axis=0)
    assert np.max(np.abs(f64(P) - P_o)) <= P_TOL


@pytest.mark.parametrize("name,T", [("tiny", 64), ("mixtral_decode", 256), ("mixtral_prefill", 3000),
                                    ("mixtral_prefill", 5000),  # past 4096 tokens: logits GEMM + top-K at E = 8
                                    ("qwen_capacity", 1000), ("deepseek_bias", 700)])
def test_route_fused_vs_oracle(name, T):
    d = dev()
    wl = synth.get_workload(name)
    x = synth.make_x(wl, device=d)[:T].contiguous()
    Wr = synth.make_router(wl, device=d)
    E, K = wl.E, wl.K
    bias = _bias(E, 7, 0.05).to(d) if wl.use_bias else None
    dims = abi.Dims(T, wl.d_model, wl.d_ff, E, K, wl.capacity_factor)
    ws = abi.alloc_workspace(dims)
    logits = torch.empty(T, E, dtype=torch.float32, device=d)
    idx = torch.empty(T, K, dtype=torch.int32, device=d)
    w = torch.empty(T, K, dtype=torch.float32, device=d)
    P = torch.empty(E, dtype=torch.float32, device=d)
    abi.moe_route(dims, x, Wr, bias, logits, idx, w, P, ws)
    torch.cuda.synchronize()
    x64, Wr64 = f64(x), f64(Wr)
    l64 = O.router_logits(x64, Wr64)
    # fp32 accumulation bound; x2 covers tensor-core accumulation (non-RNE adds)
    bound = 2.0 * O.dot_error_bound(x64, Wr64) + np.abs(l64) * 2.0 ** -23
    lg = f64(logits)
    assert np.all(np.abs(lg - l64) <= bound), float(np.max(np.abs(lg - l64) - bound))
    b32 = None if bias is None else bias.cpu().numpy()
    idx_o, w_o, _ = O.route_from_logits_f32(l64.astype(np.float32), K, b32)
    amb = ambiguous_tokens(l64, bound, K, b32)
    ig = idx.cpu().numpy()
    # exact where the worst-case bound leaves one answer; valid everywhere;
    # and in practice (errors far below the worst case) nearly always equal
    assert np.array_equal(ig[~amb], idx_o[~amb])
    assert np.mean(np.all(ig == idx_o, axis=1)) >= 0.995
    check_routing_validity(ig, l64, bound, K, b32)
    # bit-exact: the oracle's fp32 top-K on the library's own fp32 logits (and
    # bias) selects exactly the library's experts; the weights agree within the
    # fp32-vs-fp64 exp tolerance
    idx_s, w_s, _ = O.route_from_logits_f32(logits.cpu().numpy(), K, b32)
    assert np.array_equal(ig, idx_s)
    assert np.max(np.abs(f64(w) - w_s)) <= W_TOL
    wt = np.max(2 * bound, axis=1, keepdims=True) + W_TOL
    assert np.all(np.abs(f64(w)[~amb] - w_o[~amb]) <= wt[~amb])
    P_o = O.softmax_rows(l64).mean(axis=0)
    assert np.max(np.abs(f64(P) - P_o)) <= P_TOL + 2 * float(bound.max())
