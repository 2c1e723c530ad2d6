"""Chunked MoE (the layer over a batch in token chunks) against the whole-batch
layer and the fp64 oracle."""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from tests.gpu_util import (Y_MAX_ABS, Y_REL_L2, LayerInputs, assert_close_y, dev, f64, oracle_layer,
                            uncertain_tokens)

pytestmark = pytest.mark.gpu

STATS = ("counts", "f", "P", "aux", "P_topk", "aux_topk", "z_loss")


def _outs(T, E, K):
    d = dev()
    i32 = dict(dtype=torch.int32, device=d)
    f32 = dict(dtype=torch.float32, device=d)
    return dict(topk_idx=torch.empty(T, K, **i32), topk_w=torch.empty(T, K, **f32), counts=torch.empty(E, **i32),
                kept=torch.empty(E, **i32), n_dropped=torch.full((1,), -1, **i32), f=torch.empty(E, **f32),
                P=torch.empty(E, **f32), aux=torch.empty(1, **f32), P_topk=torch.empty(E, **f32),
                aux_topk=torch.empty(1, **f32), z_loss=torch.empty(1, **f32))


@pytest.mark.parametrize("name,T,chunk,ntok", [
    ("mixtral_prefill", 3000, 1024, 24),   # three chunks, the last one shorter
    ("mixtral_decode", 256, 100, 16),      # decode-sized chunks (weight-major tiles, reduction splits)
    ("deepseek_bias", 600, 256, 10),       # bias update over the whole batch
    ("tiny", 64, 64, 64),                  # one chunk = the whole batch
])
def test_chunked_matches_whole_batch_and_oracle(name, T, chunk, ntok):
    inp = LayerInputs(synth.get_workload(name), T=T)
    wl = inp.wl
    E, K, d = wl.E, wl.K, wl.d_model
    alpha = float(wl.alpha) if wl.use_bias else 0.0
    b0 = (synth.normal_f32(E, 9, synth.STREAM_MISC) * 0.05).to(dev()) if wl.use_bias else None

    bias_a = None if b0 is None else b0.clone()
    outs_a = _outs(T, E, K)
    y_a = torch.full((T, d), float("nan"), dtype=torch.float32, device=dev())
    abi.moe_layer_forward(inp.dims, inp.x, inp.Wr, bias_a, alpha, inp.W13p, inp.W2p, y_a, inp.ws, outs_a)

    bias_b = None if b0 is None else b0.clone()
    outs_b = _outs(T, E, K)
    y_b = torch.full((T, d), float("nan"), dtype=torch.float32, device=dev())
    ws_c = abi.alloc_chunked_workspace(inp.dims, chunk)
    abi.moe_reset_device_status(ws_c)
    abi.moe_layer_forward_chunked(inp.dims, chunk, inp.x, inp.Wr, bias_b, alpha, inp.W13p, inp.W2p, y_b, ws_c,
                                  outs_b)
    torch.cuda.synchronize()
    st, detail = abi.moe_get_device_status(ws_c)
    assert st == abi.MOE_OK, f"device wait ran out (code {detail})"

    # routing, statistics and the bias update are the whole batch's, bit for bit
    for key in ("topk_idx", "topk_w") + STATS:
        assert torch.equal(outs_a[key], outs_b[key]), key
    assert torch.equal(outs_b["kept"], outs_b["counts"]) and int(outs_b["n_dropped"].item()) == 0
    if b0 is not None:
        assert torch.equal(bias_a, bias_b)
    # y: the same layer up to floating-point reordering of the expert GEMMs
    ya, yb = f64(y_a), f64(y_b)
    assert np.all(np.isfinite(yb))
    assert np.max(np.abs(ya - yb)) <= 1e-3 and np.linalg.norm(ya - yb) <= 1e-5 * np.linalg.norm(ya)
    # and against the fp64 oracle on sampled tokens
    tokens = sorted(set(np.linspace(0, T - 1, ntok).astype(int).tolist()))
    b32 = None if b0 is None else b0.cpu().numpy()
    ref = oracle_layer(inp, bias32=b32, tokens=tokens)
    unc = uncertain_tokens(outs_b["topk_idx"].cpu().numpy(), ref["idx"], E, ref["capacity"])
    rows = np.asarray(tokens)
    rows = rows[~unc[rows]]
    assert len(rows) >= len(tokens) - 1
    assert_close_y(yb[rows], ref["y"][rows], Y_MAX_ABS, Y_REL_L2, "y (chunked)")


def test_chunked_bf16_output_is_rne_of_fp32():
    inp = LayerInputs(synth.get_workload("mixtral_decode"), T=300)
    T, d = inp.T, inp.wl.d_model
    ws = abi.alloc_chunked_workspace(inp.dims, 128)
    y32 = torch.empty(T, d, dtype=torch.float32, device=dev())
    y16 = torch.empty(T, d, dtype=torch.bfloat16, device=dev())
    abi.moe_layer_forward_chunked(inp.dims, 128, inp.x, inp.Wr, None, 0.0, inp.W13p, inp.W2p, y32, ws)
    abi.moe_layer_forward_chunked(inp.dims, 128, inp.x, inp.Wr, None, 0.0, inp.W13p, inp.W2p, y16, ws)
    torch.cuda.synchronize()
    assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))
