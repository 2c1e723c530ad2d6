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


def _permute_all(dims, idx, x, T, E, K, dm):
    d = dev()
    ws = abi.alloc_workspace(dims)
    i32 = dict(dtype=torch.int32, device=d)
    b = dict(counts=torch.empty(E, **i32), kept=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
             inv=torch.empty(T, K, **i32), src=torch.full((T * K,), -7, **i32),
             xp=None if x is None else torch.zeros(T * K, dm, dtype=torch.bfloat16, device=d),
             nd=torch.empty(1, **i32))
    abi.moe_reset_device_status(ws)
    abi.moe_permute(dims, idx, x, b["counts"], b["kept"], b["offsets"], b["inv"], b["src"], b["xp"], b["nd"], ws)
    torch.cuda.synchronize()
    return b, abi.moe_get_device_status(ws)


@pytest.mark.parametrize("T,E,K,cf,with_x", [(700, 8, 2, 0.0, True), (700, 16, 4, 1.0, False),
                                             (3000, 60, 4, 1.0, True), (2100, 256, 8, 0.0, False)])
def test_permute_repeated_expert_in_a_token(T, E, K, cf, with_x):
    """A token that lists an expert twice is two assignments, ranked in slot
    order: the oracle's scan over (t, k) pairs gives the expected result."""
    d = dev()
    idx_h = synth.distinct_choices(T, E, K, seed=T + 3 * E).numpy().copy()
    idx_h[::5, K - 1] = idx_h[::5, 0]          # every 5th token repeats its first expert
    idx_h[1::9, :] = idx_h[1::9, :1]            # every 9th token lists one expert K times
    idx = torch.from_numpy(idx_h).to(d)
    dm = 64
    x = synth.normal_bf16((T, dm), seed=6, stream=synth.STREAM_X, device=d) if with_x else None
    dims = abi.Dims(T, dm, 64, E, K, cf)
    b, (st, _) = _permute_all(dims, idx, x, T, E, K, dm)
    assert st == abi.MOE_OK
    o = O.dispatch(idx_h, E, O.capacity(T, K, E, cf))
    for key, ref in (("counts", "counts"), ("kept", "kept"), ("offsets", "offsets"), ("inv", "inv")):
        assert np.array_equal(b[key].cpu().numpy(), o[ref]), key
    n = int(o["offsets"][-1])
    assert np.array_equal(b["src"].cpu().numpy()[:n], o["src"])
    assert int(b["nd"].item()) == o["n_dropped"]
    if with_x:
        xs = x.view(torch.int16).cpu().numpy()
        assert np.array_equal(b["xp"].view(torch.int16).cpu().numpy()[:n], xs[o["src"]])


@pytest.mark.parametrize("T,E,K,cf,with_x", [(500, 8, 2, 0.0, True), (500, 60, 4, 1.0, False),
                                             (5000, 60, 4, 1.0, True), (3000, 256, 8, 0.0, False)])
def test_permute_skips_out_of_range_experts(T, E, K, cf, with_x):
    """Entries outside [0, E) are skipped (not counted, inv = -1) and the
    status flag reads MOE_EINDEX.  Expected values: the oracle's dispatch
    with those entries sent to an extra last expert E, whose rows come after
    every real expert's, with the capacity of the real E."""
    d = dev()
    idx_h = synth.distinct_choices(T, E, K, seed=2 * T + E).numpy().copy()
    bad = np.zeros((T, K), bool)
    bad[::11, 0] = True
    bad[3::13, K - 1] = True
    vals = np.array([E, -1, E + 1000, -2 ** 31, 2 ** 31 - 1], np.int64)
    idx_h[bad] = vals[np.arange(bad.sum()) % len(vals)]
    idx = torch.from_numpy(idx_h.astype(np.int32)).to(d)
    dm = 64
    x = synth.normal_bf16((T, dm), seed=8, stream=synth.STREAM_X, device=d) if with_x else None
    dims = abi.Dims(T, dm, 64, E, K, cf)
    b, (st, detail) = _permute_all(dims, idx, x, T, E, K, dm)
    assert st == abi.MOE_EINDEX and detail == 7
    sink = np.where(bad, E, idx_h)
    C = O.capacity(T, K, E, cf)
    o = O.dispatch(sink, E + 1, C)
    assert np.array_equal(b["counts"].cpu().numpy(), o["counts"][:E])
    assert np.array_equal(b["kept"].cpu().numpy(), o["kept"][:E])
    assert np.array_equal(b["offsets"].cpu().numpy(), o["offsets"][:E + 1])
    inv_ref = np.where(bad, -1, o["inv"])
    assert np.array_equal(b["inv"].cpu().numpy(), inv_ref)
    n = int(o["offsets"][E])
    assert np.array_equal(b["src"].cpu().numpy()[:n], o["src"][:n])
    assert np.all(b["src"].cpu().numpy()[n:] == -7)
    drops = int(np.sum(np.maximum(0, o["counts"][:E] - (C if C is not None else 1 << 40))))
    assert int(b["nd"].item()) == drops
    if with_x:
        xs = x.view(torch.int16).cpu().numpy()
        assert np.array_equal(b["xp"].view(torch.int16).cpu().numpy()[:n], xs[o["src"][:n]])
