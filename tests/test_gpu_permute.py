"""Dispatch parity: counts, capacity, offsets, ranks, drops and row gather, bit for bit."""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O
from tests.gpu_util import dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,K,cf,skew", [
    (1, 1, 1, 0.0, 0.0), (1000, 8, 2, 0.0, 0.0), (1000, 8, 2, 1.0, 1.5), (8192, 60, 4, 1.0, 2.0),
    (4096, 256, 8, 0.0, 1.1), (300, 3, 3, 0.5, 0.0), (2049, 16, 16, 1.25, 0.5), (257, 5, 2, 0.0625, 0.0),
    (16384, 8, 2, 0.0, 0.3),
    # batches of at most 1024 tokens with a gather take the one-launch dispatch
    (1024, 256, 16, 0.0, 0.7), (1024, 256, 16, 0.5, 1.0), (513, 33, 7, 0.9, 0.4)])
def test_permute_bitexact(T, E, K, cf, skew):
    d = dev()
    wts = None
    if skew > 0:
        wts = torch.tensor([(r + 1.0) ** -skew for r in range(E)])
    idx = synth.distinct_choices(T, E, K, seed=T * 31 + E, weights=wts).to(d)
    dm = 64
    x = synth.normal_bf16((T, dm), seed=5, stream=synth.STREAM_X, device=d)
    dims = abi.Dims(T, dm, 64, E, K, cf)
    ws = abi.alloc_workspace(dims)
    i32 = dict(dtype=torch.int32, device=d)
    counts, kept = torch.empty(E, **i32), torch.empty(E, **i32)
    offsets, inv = torch.empty(E + 1, **i32), torch.empty(T, K, **i32)
    src = torch.full((T * K,), -7, **i32)
    xp = torch.zeros(T * K, dm, dtype=torch.bfloat16, device=d)
    nd = torch.empty(1, **i32)
    abi.moe_permute(dims, idx, x, counts, kept, offsets, inv, src, xp, nd, ws)
    torch.cuda.synchronize()
    C = O.capacity(T, K, E, cf)
    o = O.dispatch(idx.cpu().numpy(), E, C)
    assert np.array_equal(counts.cpu().numpy(), o["counts"])
    assert np.array_equal(kept.cpu().numpy(), o["kept"])
    assert np.array_equal(offsets.cpu().numpy(), o["offsets"])
    assert np.array_equal(inv.cpu().numpy(), o["inv"])
    n = int(o["offsets"][-1])
    assert np.array_equal(src.cpu().numpy()[:n], o["src"])
    assert np.all(src.cpu().numpy()[n:] == -7)          # rows past N_kept untouched
    assert int(nd.item()) == o["n_dropped"]
    xs = x.view(torch.int16).cpu().numpy()
    assert np.array_equal(xp.view(torch.int16).cpu().numpy()[:n], xs[o["src"]])


def test_permute_is_deterministic():
    d = dev()
    T, E, K = 5000, 32, 4
    idx = synth.distinct_choices(T, E, K, seed=3).to(d)
    dims = abi.Dims(T, 64, 64, E, K, 0.9)
    ws = abi.alloc_workspace(dims)
    outs = []
    for _ in range(3):
        i32 = dict(dtype=torch.int32, device=d)
        bufs = [torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32),
                torch.empty(T, K, **i32), torch.full((T * K,), -1, **i32), torch.empty(1, **i32)]
        abi.moe_permute(dims, idx, None, bufs[0], bufs[1], bufs[2], bufs[3], bufs[4], None, bufs[5], ws)
        outs.append([b.cpu() for b in bufs])
    for b in range(6):
        assert torch.equal(outs[0][b], outs[1][b]) and torch.equal(outs[0][b], outs[2][b])
