"""moe_permute_noalloc: dispatch for callers that cannot allocate.

Some callers cannot give the library a workspace: a host runtime that owns
every device buffer and exposes no allocator to its plug-ins, or a serving
loop that may not allocate (or synchronise the device, as an allocator can)
between steps.  For them the dispatch step has a variant whose scratch is a
fixed array inside the library.  These tests call it through the C ABI and
check it against the workspace version, bit for bit, on two calls in a row
(the shared scratch keeps the previous call's contents, which must not leak
into the next result).

This file is collected last so that a stop-at-first-failure run has already
run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, synth

pytestmark = pytest.mark.gpu


def _buffers(T, E, K, d, dev):
    i32 = dict(dtype=torch.int32, device=dev)
    return dict(counts=torch.full((E,), -9, **i32), kept=torch.full((E,), -9, **i32),
                offsets=torch.full((E + 1,), -9, **i32), inv=torch.full((T, K), -9, **i32),
                src=torch.full((T * K,), -9, **i32), x_perm=torch.zeros(T * K, d, dtype=torch.bfloat16, device=dev),
                n_dropped=torch.full((1,), -9, **i32))


def _run(fn, dims, idx, x, b, ws=None):
    args = (dims, idx, x, b["counts"], b["kept"], b["offsets"], b["inv"], b["src"], b["x_perm"], b["n_dropped"])
    if ws is None:
        fn(*args)
    else:
        fn(*args, ws)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T,E,K,cf,d", [(5000, 60, 4, 1.0, 64), (3000, 256, 8, 0.0, 128), (700, 8, 2, 0.0, 256)])
def test_noalloc_matches_workspace_dispatch_twice(T, E, K, cf, d):
    dev = torch.device("cuda", 0)
    dims = abi.Dims(T, d, 64, E, K, cf)
    ws = abi.alloc_workspace(dims)
    for call in range(2):   # a second call sees the first call's leftovers in the shared scratch
        wts = torch.tensor([(r + 1.0) ** -(0.5 + call) for r in range(E)])
        idx = synth.distinct_choices(T, E, K, seed=100 * call + T, weights=wts).to(dev)
        x = synth.normal_bf16((T, d), 7 + call, synth.STREAM_X, 1.0, dev)
        ref = _buffers(T, E, K, d, dev)
        got = _buffers(T, E, K, d, dev)
        _run(abi.moe_permute, dims, idx, x, ref, ws)
        _run(abi.moe_permute_noalloc, dims, idx, x, got)
        n = int(ref["offsets"][-1].item())
        for key in ("counts", "kept", "offsets", "inv", "n_dropped"):
            assert torch.equal(got[key], ref[key]), (call, key)
        assert torch.equal(got["src"][:n], ref["src"][:n]), call
        assert torch.equal(got["x_perm"][:n].view(torch.int16), ref["x_perm"][:n].view(torch.int16)), call


def test_noalloc_rejects_batches_beyond_its_scratch():
    dev = torch.device("cuda", 0)
    T, E, K = 70000, 256, 8          # ceil(70000 / 256) * 256 = 70144 > 65536
    dims = abi.Dims(T, 64, 64, E, K)
    b = _buffers(4, E, K, 64, dev)   # never touched: the size check comes first
    idx = torch.zeros(4, K, dtype=torch.int32, device=dev)
    with pytest.raises(abi.MoEError) as e:
        abi.moe_permute_noalloc(dims, idx, None, b["counts"], b["kept"], b["offsets"], b["inv"], b["src"], None,
                                None)
    assert e.value.status == abi.MOE_ESCRATCH
