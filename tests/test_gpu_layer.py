"""Whole-layer parity: moe_layer_forward against the fp64 oracle."""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O
from tests.gpu_util import (Y_MAX_ABS, Y_MIRROR_MAX_ABS, Y_MIRROR_REL_L2, Y_REL_L2, LayerInputs, ambiguous_tokens,
                            assert_close_y, check_routing_validity, covering_sample, dev, experts_compared, f64,
                            oracle_layer, uncertain_tokens)

pytestmark = pytest.mark.gpu


def _forward(inp: LayerInputs, bias=None, alpha=0.0):
    d = dev()
    T, E, K = inp.T, inp.wl.E, inp.wl.K
    i32 = dict(dtype=torch.int32, device=d)
    outs = dict(topk_idx=torch.empty(T, K, **i32), topk_w=torch.empty(T, K, dtype=torch.float32, device=d),
                logits=torch.empty(T, E, dtype=torch.float32, device=d), counts=torch.empty(E, **i32),
                kept=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32), inv=torch.empty(T, K, **i32),
                n_dropped=torch.empty(1, **i32), f=torch.empty(E, dtype=torch.float32, device=d),
                P=torch.empty(E, dtype=torch.float32, device=d), aux=torch.empty(1, dtype=torch.float32, device=d),
                P_topk=torch.empty(E, dtype=torch.float32, device=d),
                aux_topk=torch.empty(1, dtype=torch.float32, device=d),
                z_loss=torch.empty(1, dtype=torch.float32, device=d))
    y = torch.full((T, inp.wl.d_model), float("nan"), dtype=torch.float32, device=d)
    abi.moe_reset_device_status(inp.ws)
    abi.moe_layer_forward(inp.dims, inp.x, inp.Wr, bias, alpha, inp.W13p, inp.W2p, y, inp.ws, outs)
    torch.cuda.synchronize()
    st, detail = abi.moe_get_device_status(inp.ws)
    assert st == abi.MOE_OK, f"device wait ran out (code {detail})"
    return y, outs


def _check(inp, y, outs, ref, bias32=None, tokens=None, mirror=None):
    K, E = inp.wl.K, inp.wl.E
    x64, Wr64 = inp.host()
    l64 = ref["logits"]
    bound = 2.0 * O.dot_error_bound(x64, Wr64) + np.abs(l64) * 2.0 ** -23
    ig = outs["topk_idx"].cpu().numpy()
    check_routing_validity(ig, l64, bound, K, bias32)
    amb = ambiguous_tokens(l64, bound, K, bias32)
    assert np.array_equal(ig[~amb], ref["idx"][~amb])
    unc = uncertain_tokens(ig, ref["idx"], E, ref["capacity"])
    assert unc.mean() <= 0.01, f"{unc.sum()} tokens routed differently"
    if not unc.any():
        assert np.array_equal(outs["counts"].cpu().numpy(), ref["counts"])
        assert np.array_equal(outs["offsets"].cpu().numpy(), ref["offsets"])
        assert np.array_equal(outs["inv"].cpu().numpy(), ref["inv"])
        assert int(outs["n_dropped"].item()) == ref["n_dropped"]
    rows = np.arange(inp.T) if tokens is None else np.asarray(tokens)
    rows = rows[~unc[rows]]
    yg = f64(y)
    assert_close_y(yg[rows], ref["y"][rows], Y_MAX_ABS, Y_REL_L2, "y")
    if mirror is not None:
        assert_close_y(yg[rows], mirror["y"][rows], Y_MIRROR_MAX_ABS, Y_MIRROR_REL_L2, "y (H rounded)")
    # statistics
    cg = outs["counts"].cpu().numpy()
    assert cg.sum() == inp.T * K
    f_ref = cg / float(inp.T * K)
    assert np.allclose(f64(outs["f"]), f_ref, atol=1e-7)
    assert np.max(np.abs(f64(outs["P"]) - ref["P"])) <= 1e-5 + 2 * float(bound.max())
    aux_ref = E * float(np.sum(f_ref * ref["P"]))
    assert abs(float(outs["aux"].item()) - aux_ref) <= 1e-4 * max(1.0, aux_ref)
    # top-K-only balance statistic: a token routed differently moves P~ by at most 2/T
    Pt = f64(outs["P_topk"])
    assert abs(Pt.sum() - 1.0) <= 1e-5
    assert np.max(np.abs(Pt - ref["P_topk"])) <= 1e-5 + 2.0 * unc.sum() / inp.T
    at_ref = E * float(np.sum(f_ref * Pt))
    assert abs(float(outs["aux_topk"].item()) - at_ref) <= 1e-5 * max(1.0, at_ref)
    # router z-loss: each log-sum-exp moves by at most the largest logit error
    l64m = l64.max(axis=1)
    lse = l64m + np.log(np.exp(l64 - l64m[:, None]).sum(axis=1))
    delta = float(bound.max()) + 2e-6 * float(np.abs(lse).max())
    tol = 2.0 * float(np.abs(lse).max()) * delta + delta * delta + 1e-5 * ref["z_loss"]
    assert abs(float(outs["z_loss"].item()) - ref["z_loss"]) <= tol
    return rows


def test_layer_tiny_full():
    inp = LayerInputs(synth.get_workload("tiny"))
    y, outs = _forward(inp)
    ref = oracle_layer(inp)
    mirror = oracle_layer(inp, h_round=O.bf16_round)
    rows = _check(inp, y, outs, ref, mirror=mirror)
    assert len(rows) == inp.T


@pytest.mark.parametrize("name,T,ntok", [
    ("mixtral_decode", 256, 24), ("mixtral_decode", 37, 37), ("mixtral_prefill", 1500, 24),
    ("qwen_capacity", 2000, 48), ("qwen_capacity", 700, 32), ("deepseek_bias", 600, 12)])
def test_layer_reduced_T(name, T, ntok):
    inp = LayerInputs(synth.get_workload(name), T=T)
    bias = None
    b32 = None
    if inp.wl.use_bias:
        bias = (synth.normal_f32(inp.wl.E, 9, synth.STREAM_MISC) * 0.05).to(dev())
        b32 = bias.cpu().numpy()
    y, outs = _forward(inp, bias)
    tokens = sorted(set(np.linspace(0, T - 1, ntok).astype(int).tolist()))
    ref = oracle_layer(inp, bias32=b32, tokens=tokens)
    _check(inp, y, outs, ref, bias32=b32, tokens=tokens)


def test_layer_all_tokens_one_expert():
    """Degenerate routing: every token picks expert 0 first (a huge bias)."""
    wl = synth.get_workload("tiny")
    inp = LayerInputs(wl)
    bias = torch.zeros(wl.E, dtype=torch.float32, device=dev())
    bias[0] = 1e4
    y, outs = _forward(inp, bias)
    assert outs["counts"][0].item() == inp.T
    ref = oracle_layer(inp, bias32=bias.cpu().numpy())
    _check(inp, y, outs, ref, bias32=bias.cpu().numpy())


def test_layer_bias_update_in_place():
    wl = synth.get_workload("tiny")
    inp = LayerInputs(wl)
    bias = torch.zeros(wl.E, dtype=torch.float32, device=dev())
    y, outs = _forward(inp, bias, alpha=1e-3)
    ref = oracle_layer(inp, bias32=np.zeros(wl.E, np.float32), alpha=1e-3)
    assert np.array_equal(outs["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(bias.cpu().numpy().view(np.uint32), ref["bias"].view(np.uint32))


@pytest.mark.parametrize("name,S", [("mixtral_decode", 256), ("mixtral_prefill", 512), ("qwen_capacity", 512),
                                    ("deepseek_bias", 512)])
def test_layer_full_size_sampled(name, S):
    """Each workload at its full size, in the launch configuration bench.py
    times.  The fp64 oracle evaluates every token of the decode batch, and
    at the larger shapes a seeded sample of 512 tokens chosen so that every
    expert with kept rows holds a compared row (routing, counts and capacity
    always over the whole batch)."""
    inp = LayerInputs(synth.get_workload(name))
    T = inp.T
    bias = b32 = None
    if inp.wl.use_bias:
        bias = torch.zeros(inp.wl.E, dtype=torch.float32, device=dev())
        b32 = np.zeros(inp.wl.E, np.float32)
    y, outs = _forward(inp, bias)
    if S >= T:
        tokens = list(range(T))
        need = None
    else:
        tokens, need = covering_sample(inp, S, b32, seed=S + T)
    ref = oracle_layer(inp, bias32=b32, tokens=tokens)
    rows = _check(inp, y, outs, ref, bias32=b32, tokens=tokens)
    assert len(rows) >= len(tokens) - max(2, len(tokens) // 100)
    if need is not None:
        assert experts_compared(rows, ref["idx"], ref["inv"]) == need
    # every token's output is finite and dropped-everything tokens are exactly 0
    yg = f64(y)
    assert np.all(np.isfinite(yg))
    inv = outs["inv"].cpu().numpy()
    dead = np.all(inv < 0, axis=1)
    assert np.all(yg[dead] == 0)


@pytest.mark.parametrize("name,T", [("tiny", 64), ("mixtral_decode", 256), ("qwen_capacity", 1000),
                                    ("deepseek_bias", 300)])
def test_layer_bf16_output_is_rne_of_fp32(name, T):
    """The bf16 layer output is, bit for bit, the round-to-nearest-even of the
    fp32 output of the same call (every step is deterministic)."""
    inp = LayerInputs(synth.get_workload(name), T=T)
    d = dev()
    y32 = torch.empty(T, inp.wl.d_model, dtype=torch.float32, device=d)
    y16 = torch.empty(T, inp.wl.d_model, dtype=torch.bfloat16, device=d)
    abi.moe_layer_forward(inp.dims, inp.x, inp.Wr, None, 0.0, inp.W13p, inp.W2p, y32, inp.ws)
    abi.moe_layer_forward(inp.dims, inp.x, inp.Wr, None, 0.0, inp.W13p, inp.W2p, y16, inp.ws)
    torch.cuda.synchronize()
    assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
