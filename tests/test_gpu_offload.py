"""Expert offloading on the GPU: INT4 packing and unpacking into cache slots,
the slot-indirected expert GEMMs, and the offloaded layer over several steps.

Expected values: the oracle's INT4 quantization and dequantization of the
same weights (laid out by moe_pack_weights, itself checked element by element
elsewhere), the oracle layer on the dequantized weights, and the oracle's LRU
cache and prediction on the oracle's own routing.
"""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from moe_layer_gemm_b200.offload import OffloadedLayer, quantize_experts_to_host
from oracle import moe_oracle as O
from tests.gpu_util import Y_MAX_ABS, Y_REL_L2, assert_close_y, dev, f64, uncertain_tokens

pytestmark = pytest.mark.gpu


def _weights(E, d, f, seed, std=0.05):
    dv = dev()
    W1 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W1, std, dv)
    W3 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W3, std, dv)
    W2 = synth.normal_bf16((E, f, d), seed, synth.STREAM_W2, std, dv)
    return W1, W3, W2


def _dequantized(W):
    """The oracle's INT4 round trip of each expert matrix [E, K_red, N]."""
    out = np.empty(W.shape)
    for e in range(W.shape[0]):
        out[e] = O.int4_dequantize(*O.int4_quantize(f64(W[e])))
    return out


@pytest.mark.parametrize("E,d,f", [(6, 256, 128), (3, 192, 320)])
def test_int4_unpack_equals_packed_oracle_dequantization(E, d, f):
    dv = dev()
    dims = abi.Dims(1, d, f, E, 1)
    W1, W3, W2 = _weights(E, d, f, 5)
    n13, ns13, n2, ns2 = abi.moe_int4_bytes(dims)
    q13 = torch.empty(n13, dtype=torch.uint8, device=dv)
    s13 = torch.empty(ns13 // 4, dtype=torch.float32, device=dv)
    q2 = torch.empty(n2, dtype=torch.uint8, device=dv)
    s2 = torch.empty(ns2 // 4, dtype=torch.float32, device=dv)
    abi.moe_int4_pack(dims, W1, W3, W2, q13, s13, q2, s2)
    # reference: the oracle's dequantized weights in the packed layout
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).to(dv)  # noqa: E731  (exact: bf16 values)
    R13, R2 = abi.pack_weights(dims, bf(_dequantized(W1)), bf(_dequantized(W3)), bf(_dequantized(W2)))
    per13, per2 = R13.numel() // E, R2.numel() // E
    n_slots = E + 2
    slots = [(3 * e + 1) % n_slots for e in range(E)]        # a permuted placement
    for src in ("device", "host"):
        qs = (q13, s13, q2, s2) if src == "device" else tuple(t.cpu().pin_memory() for t in (q13, s13, q2, s2))
        W13c = torch.zeros(n_slots * per13, dtype=torch.bfloat16, device=dv)
        W2c = torch.zeros(n_slots * per2, dtype=torch.bfloat16, device=dv)
        abi.moe_int4_unpack(dims, list(range(E)), slots, *qs, n_slots, W13c, W2c)
        torch.cuda.synchronize()
        for e, sl in enumerate(slots):
            assert torch.equal(W13c[sl * per13:(sl + 1) * per13].view(torch.int16),
                               R13[e * per13:(e + 1) * per13].view(torch.int16)), (src, e)
            assert torch.equal(W2c[sl * per2:(sl + 1) * per2].view(torch.int16),
                               R2[e * per2:(e + 1) * per2].view(torch.int16)), (src, e)


def test_int4_unpack_refuses_pageable_host_memory():
    dims = abi.Dims(1, 128, 128, 2, 1)
    n13, ns13, n2, ns2 = abi.moe_int4_bytes(dims)
    pageable = [torch.zeros(n, dtype=torch.uint8) for n in (n13, ns13, n2, ns2)]
    per13, per2 = (b // 2 for b in abi.moe_packed_weight_bytes(dims))
    W13c = torch.zeros(per13, dtype=torch.bfloat16, device=dev())
    W2c = torch.zeros(per2, dtype=torch.bfloat16, device=dev())
    with pytest.raises(ValueError):   # the binding refuses before the call
        abi.moe_int4_unpack(dims, [0], [0], pageable[0], pageable[1].view(torch.float32), pageable[2],
                            pageable[3].view(torch.float32), 1, W13c, W2c)
    # and so does the library itself, before any launch
    import ctypes
    lib = abi.load()
    one = (ctypes.c_int32 * 1)(0)
    c = dims.c()
    st = lib.moe_int4_unpack(ctypes.byref(c), 1, one, one, *[ctypes.c_void_p(t.data_ptr()) for t in pageable], 1,
                             ctypes.c_void_p(W13c.data_ptr()), ctypes.c_void_p(W2c.data_ptr()), None)
    assert st == abi.MOE_EUNSUPPORTED


@pytest.mark.parametrize("T,d,f,E,K", [(300, 256, 192, 16, 4), (256, 512, 512, 8, 2), (2048, 256, 256, 4, 2)])
def test_slot_indirected_ffn_equals_ffn(T, d, f, E, K):
    """The same weights moved to permuted cache slots give bit-identical
    expert outputs (only the weight addresses change)."""
    dv = dev()
    dims = abi.Dims(T, d, f, E, K)
    W1, W3, W2 = _weights(E, d, f, 9)
    W13p, W2p = abi.pack_weights(dims, W1, W3, W2)
    per13, per2 = W13p.numel() // E, W2p.numel() // E
    n_slots = E + 3
    slot = [(5 * e + 2) % n_slots for e in range(E)]
    W13c = torch.zeros(n_slots * per13, dtype=torch.bfloat16, device=dv)
    W2c = torch.zeros(n_slots * per2, dtype=torch.bfloat16, device=dv)
    for e, sl in enumerate(slot):
        W13c[sl * per13:(sl + 1) * per13] = W13p[e * per13:(e + 1) * per13]
        W2c[sl * per2:(sl + 1) * per2] = W2p[e * per2:(e + 1) * per2]
    idx = synth.distinct_choices(T, E, K, seed=T, weights=torch.tensor([(r + 1.0) ** -0.8 for r in range(E)])).to(dv)
    x = synth.normal_bf16((T, d), 4, synth.STREAM_X, 1.0, dv)
    ws = abi.alloc_workspace(dims)
    i32 = dict(dtype=torch.int32, device=dv)
    A = T * K
    counts, kept, offsets = torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32)
    inv, src = torch.empty(T, K, **i32), torch.empty(A, **i32)
    xp = torch.zeros(A, d, dtype=torch.bfloat16, device=dv)
    abi.moe_permute(dims, idx, x, counts, kept, offsets, inv, src, xp, None, ws)
    h1, h2 = (torch.zeros(A, f, dtype=torch.bfloat16, device=dv) for _ in range(2))
    y1, y2 = (torch.zeros(A, d, dtype=torch.float32, device=dv) for _ in range(2))
    abi.moe_expert_ffn(dims, xp, offsets, W13p, W2p, h1, y1, ws)
    abi.moe_expert_ffn_slots(dims, xp, offsets, torch.tensor(slot, **i32), n_slots, W13c, W2c, h2, y2, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_status(ws)[0] == abi.MOE_OK
    n = int(offsets[-1].item())
    assert torch.equal(h1[:n].view(torch.int16), h2[:n].view(torch.int16))
    assert torch.equal(y1[:n].view(torch.int32), y2[:n].view(torch.int32))


@pytest.mark.parametrize("T,d,f,E,K", [(300, 256, 192, 16, 4), (512, 512, 512, 16, 4), (256, 512, 512, 8, 2)])
def test_skipped_experts_then_complement_equal_one_call(T, d, f, E, K):
    """Two calls with complementary slot tables (MOE_SLOT_SKIP for the experts
    the other call covers) write the same h and y_perm as one call with all
    experts: a skipped expert's rows are left alone, the others are computed
    exactly as before."""
    dv = dev()
    dims = abi.Dims(T, d, f, E, K)
    W1, W3, W2 = _weights(E, d, f, 21)
    W13p, W2p = abi.pack_weights(dims, W1, W3, W2)
    idx = synth.distinct_choices(T, E, K, seed=T + 1, weights=torch.tensor([(r + 1.0) ** -1.2 for r in range(E)])).to(dv)
    x = synth.normal_bf16((T, d), 6, synth.STREAM_X, 1.0, dv)
    ws = abi.alloc_workspace(dims)
    i32 = dict(dtype=torch.int32, device=dv)
    A = T * K
    counts, kept, offsets = torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32)
    inv, src = torch.empty(T, K, **i32), torch.empty(A, **i32)
    xp = torch.zeros(A, d, dtype=torch.bfloat16, device=dv)
    abi.moe_permute(dims, idx, x, counts, kept, offsets, inv, src, xp, None, ws)
    ident = torch.arange(E, **i32)
    h1, h2 = (torch.zeros(A, f, dtype=torch.bfloat16, device=dv) for _ in range(2))
    y1, y2 = (torch.zeros(A, d, dtype=torch.float32, device=dv) for _ in range(2))
    abi.moe_expert_ffn_slots(dims, xp, offsets, ident, E, W13p, W2p, h1, y1, ws)
    odd = torch.arange(E, device=dv) % 2 == 1
    first = torch.where(odd, torch.full_like(ident, abi.MOE_SLOT_SKIP), ident)
    second = torch.where(odd, ident, torch.full_like(ident, abi.MOE_SLOT_SKIP))
    abi.moe_expert_ffn_slots(dims, xp, offsets, first, E, W13p, W2p, h2, y2, ws)
    torch.cuda.synchronize()
    n = int(offsets[-1].item())
    off = offsets.cpu().numpy()
    # after the first call the odd experts' rows are untouched (still zero)
    for e in range(1, E, 2):
        assert torch.count_nonzero(y2[off[e]:off[e + 1]]) == 0
    abi.moe_expert_ffn_slots(dims, xp, offsets, second, E, W13p, W2p, h2, y2, ws)
    torch.cuda.synchronize()
    assert abi.moe_get_device_status(ws)[0] == abi.MOE_OK
    assert torch.equal(h1[:n].view(torch.int16), h2[:n].view(torch.int16))
    assert torch.equal(y1[:n].view(torch.int32), y2[:n].view(torch.int32))


def test_offloaded_layer_steps_match_oracle():
    """Eight decode-sized steps (fresh tokens each) with 16 experts in host
    memory and 10 cache slots, 3 predicted experts loaded ahead per step."""
    dv = dev()
    T, d, f, E, K, slots, width = 8, 256, 128, 16, 1, 10, 3
    dims = abi.Dims(T, d, f, E, K)
    W1, W3, W2 = _weights(E, d, f, 13)
    Wr = synth.normal_bf16((d, E), 13, synth.STREAM_WR, 0.05, dv)
    q = quantize_experts_to_host(dims, W1, W3, W2)
    layer = OffloadedLayer(dims, Wr, *q, n_slots=slots, prefetch=width)
    W1d, W3d, W2d = _dequantized(W1), _dequantized(W3), _dequantized(W2)
    Wr64 = f64(Wr)
    needed_o, counts_o = [], []
    for step in range(8):
        x = synth.normal_bf16((T, d), 100 + step, synth.STREAM_X, 1.0, dv)
        y = torch.full((T, d), float("nan"), dtype=torch.float32, device=dv)
        layer.forward(x, y)
        torch.cuda.synchronize()
        assert abi.moe_get_device_status(layer.ws)[0] == abi.MOE_OK
        ref = O.moe_layer(f64(x), Wr64, W1d, W3d, W2d, K)
        unc = uncertain_tokens(layer.idx.cpu().numpy(), ref["idx"], E, None)
        assert not unc.any()
        assert_close_y(f64(y), ref["y"], Y_MAX_ABS, Y_REL_L2, f"step {step}")
        needed_o.append([int(e) for e in np.nonzero(ref["kept"])[0]])
        counts_o.append(ref["counts"])
    preds = O.routing_history_prediction(counts_o, width)
    plan = O.lru_expert_cache(needed_o, slots, preds)
    for t, rec in enumerate(layer.log):
        assert rec["needed"] == needed_o[t]
        assert rec["loads"] == plan[t]["loads"] and rec["prefetch_loads"] == plan[t]["prefetch_loads"], t
        assert rec["hits"] == plan[t]["hits"] and rec["prefetch_hits"] == plan[t]["prefetch_hits"], t
