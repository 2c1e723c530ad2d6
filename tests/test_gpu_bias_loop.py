"""Aux-free balancing loop: route with bias -> count -> update, 10 steps."""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O
from tests.gpu_util import LayerInputs, dev

pytestmark = pytest.mark.gpu


def test_bias_loop_bitexact_on_shared_logits():
    """Same fp32 logits on both sides each step: selections, counts and the
    bias after every one of 10 steps agree bit for bit."""
    d = dev()
    T, E, K, alpha = 4096, 256, 8, 1e-3
    dims = abi.Dims(T, 128, 128, E, K)
    ws = abi.alloc_workspace(dims)
    i32 = dict(dtype=torch.int32, device=d)
    bias = torch.zeros(E, dtype=torch.float32, device=d)
    b_ref = np.zeros(E, np.float32)
    scale = torch.tensor([(r + 1.0) ** -0.5 for r in range(E)], device=d) * 3.0
    for step in range(10):
        logits = (synth.logits_f32(T, E, seed=4000 + step, device=d, tie_frac=0.05) * scale).contiguous()
        idx = torch.empty(T, K, **i32)
        w = torch.empty(T, K, dtype=torch.float32, device=d)
        abi.moe_route_from_logits(dims, logits, bias, idx, w, None, ws)
        counts, kept, off = torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32)
        inv, src = torch.empty(T, K, **i32), torch.empty(T * K, **i32)
        abi.moe_permute(dims, idx, None, counts, kept, off, inv, src, None, None, ws)
        abi.moe_bias_update(dims, counts, alpha, bias)
        torch.cuda.synchronize()
        idx_o, _, _ = O.route_from_logits_f32(logits.cpu().numpy(), K, b_ref)
        c_o = O.expert_counts(idx_o, E)
        assert np.array_equal(idx.cpu().numpy(), idx_o), step
        assert np.array_equal(counts.cpu().numpy(), c_o), step
        b_ref = O.bias_update(b_ref, c_o, T, K, alpha)
        assert np.array_equal(bias.cpu().numpy().view(np.uint32), b_ref.view(np.uint32)), step
    # popular experts (large logit scale, low index) were pushed down
    assert b_ref[:8].mean() < b_ref[-8:].mean()


def test_bias_loop_layer_deepseek_shape():
    """moe_layer_forward with the in-place bias update over 10 steps of the
    DeepSeek-V3-shaped workload (fresh tokens each step): every step the
    bias moves by exactly +-alpha or 0 per expert, as its own counts say,
    and the counts agree with the oracle's routing of the same tokens."""
    wl = synth.get_workload("deepseek_bias")
    inp = LayerInputs(wl, T=1024)
    d = dev()
    E, K, T = wl.E, wl.K, inp.T
    bias = torch.zeros(E, dtype=torch.float32, device=d)
    a32 = np.float32(wl.alpha)
    i32 = dict(dtype=torch.int32, device=d)
    y = torch.empty(T, wl.d_model, dtype=torch.float32, device=d)
    for step in range(10):
        x = synth.make_x(wl, step=step, device=d)[:T].contiguous()
        before = bias.cpu().numpy().copy()
        counts = torch.empty(E, **i32)
        abi.moe_layer_forward(inp.dims, x, inp.Wr, bias, wl.alpha, inp.W13p, inp.W2p, y, inp.ws, {"counts": counts})
        torch.cuda.synchronize()
        after = bias.cpu().numpy()
        c = counts.cpu().numpy()
        assert c.sum() == T * K
        lhs = c.astype(np.int64) * E
        want = before.copy()
        want[lhs > T * K] = (before[lhs > T * K] - a32).astype(np.float32)
        want[lhs < T * K] = (before[lhs < T * K] + a32).astype(np.float32)
        assert np.array_equal(after.view(np.uint32), want.view(np.uint32)), step
        # the oracle's routing of the same tokens with the same (pre-update) bias
        x64 = x.cpu().double().numpy()
        l32 = O.router_logits(x64, inp.host()[1]).astype(np.float32)
        idx_o, _, _ = O.route_from_logits_f32(l32, K, before)
        c_o = O.expert_counts(idx_o, E)
        assert np.abs(c - c_o).sum() <= 0.01 * T * K, step
