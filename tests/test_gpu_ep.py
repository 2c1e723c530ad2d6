"""Expert parallelism on one GPU: the library's kernels in the EP step sequence.

G ranks are emulated by G host threads, each running ep_forward with
CudaSteps for its own tokens and its own block of experts.  The exchange is
an in-process stand-in for the all-to-all: each thread synchronises the
device, publishes its send buffers, and copies what the others published
(host barriers between the phases), so no kernel ever waits for another
kernel.  Checks: moe_ep_regroup against the oracle's stable grouping, bit
for bit; every rank's output against the single-GPU layer on its own tokens
(same kernels, other groupings of the rows) and against the fp64 oracle.
"""
import threading

import numpy as np
import pytest
import torch

from moe_layer_gemm_b200 import abi, ep, synth
from oracle import moe_oracle as O
from tests.gpu_util import Y_MAX_ABS, Y_REL_L2, assert_close_y, dev, f64, rel_l2, uncertain_tokens

pytestmark = pytest.mark.gpu


class Hub:
    def __init__(self, G):
        self.G = G
        self.bar = threading.Barrier(G, timeout=300)
        self.slots = [None] * G


class ThreadExchange:
    """All-to-all between threads of one process (host-synchronised copies)."""

    def __init__(self, hub, rank):
        self.hub, self.rank = hub, rank

    def _swap(self, mine, take):
        torch.cuda.synchronize()
        self.hub.slots[self.rank] = mine
        self.hub.bar.wait()
        out = take([self.hub.slots[s] for s in range(self.hub.G)])
        torch.cuda.synchronize()
        self.hub.bar.wait()
        return out

    def counts(self, send):
        El = send.numel() // self.hub.G
        r = self.rank
        return self._swap(send.clone(), lambda sl: torch.cat([s[r * El:(r + 1) * El] for s in sl]))

    def rows(self, send, s_out, s_in):
        r = self.rank
        out = self._swap(list(torch.split(send, s_out)), lambda sl: torch.cat([s[r] for s in sl]).contiguous())
        assert out.shape[0] == sum(s_in)
        return out

    def sum(self, t):
        tot = self._swap(t.clone(), lambda sl: torch.stack(sl).sum(0).to(t.dtype))
        t.copy_(tot)
        return t


def test_regroup_matches_stable_grouping():
    d = dev()
    rng = np.random.default_rng(3)
    for G, El, dm in ((1, 8, 64), (4, 2, 128), (8, 32, 64), (8, 256, 16)):
        rc = rng.integers(0, 9, size=(G, El)).astype(np.int32)
        rc[rng.random((G, El)) < 0.3] = 0
        n = int(rc.sum())
        rows = synth.normal_bf16((max(n, 1), dm), G * El, synth.STREAM_X, device=d)[:n].contiguous()
        out = torch.full((max(n, 1), dm), -7.0, dtype=torch.bfloat16, device=d)[:n]
        off = torch.full((El + 1,), -1, dtype=torch.int32, device=d)
        row_of = torch.full((max(n, 1),), -1, dtype=torch.int32, device=d)[:n]
        abi.moe_ep_regroup(G, El, torch.from_numpy(rc.reshape(-1)).to(d), rows, out, off, row_of)
        torch.cuda.synchronize()
        ids = np.concatenate([np.repeat(np.arange(El), rc[s]) for s in range(G)]).astype(np.int64)
        g = O.dispatch(ids[:, None], El)
        assert np.array_equal(off.cpu().numpy(), g["offsets"])
        assert np.array_equal(row_of.cpu().numpy(), g["inv"][:, 0])
        if n:
            assert np.array_equal(out.view(torch.int16).cpu().numpy(),
                                  rows.view(torch.int16).cpu().numpy()[g["src"]])


CASES = [
    # (tokens per rank, d, f, E, K, capacity factor, bias: hot experts or None)
    ([96, 57], 1024, 2048, 8, 2, 0.0, None),
    ([64, 33, 80, 17], 512, 1024, 16, 4, 1.0, None),
    ([40, 70, 25, 51], 256, 512, 8, 2, 0.0, [0]),
]


@pytest.mark.parametrize("case", CASES)
def test_ep_ranks_match_single_gpu_layer_and_oracle(case):
    Ts, dm, df, E, K, cf, hot = case
    G = len(Ts)
    El = E // G
    d = dev()
    T = sum(Ts)
    x = synth.normal_bf16((T, dm), 21, synth.STREAM_X, device=d)
    Wr = synth.normal_bf16((dm, E), 21, synth.STREAM_WR, 0.05, device=d)
    W1 = synth.normal_bf16((E, dm, df), 21, synth.STREAM_W1, 0.02, device=d)
    W3 = synth.normal_bf16((E, dm, df), 21, synth.STREAM_W3, 0.02, device=d)
    W2 = synth.normal_bf16((E, df, dm), 21, synth.STREAM_W2, 0.02, device=d)
    bias0 = torch.zeros(E, dtype=torch.float32, device=d)
    if hot:
        bias0[hot] = 50.0
    alpha = 1e-3
    full_dims = abi.Dims(T, dm, df, E, K)
    W13p, W2p = abi.pack_weights(full_dims, W1, W3, W2)
    local = []
    for r in range(G):
        blk = ep.expert_block(r, G, E)
        local.append(abi.pack_weights(abi.Dims(1, dm, df, El, 1), W1[blk.start:blk.stop].contiguous(),
                                      W3[blk.start:blk.stop].contiguous(), W2[blk.start:blk.stop].contiguous()))
    torch.cuda.synchronize()
    hub = Hub(G)
    ys = [torch.full((Ts[r], dm), float("nan"), dtype=torch.float32, device=d) for r in range(G)]
    biases = [bias0.clone() for _ in range(G)]
    steps = [ep.CudaSteps(abi.Dims(Ts[r], dm, df, E, K, cf), r, G, Wr, *local[r]) for r in range(G)]
    errors = [None] * G
    totals = [None] * G

    def run(r):
        try:
            torch.cuda.set_device(d)
            t0 = sum(Ts[:r])
            _, totals[r] = ep.ep_forward(steps[r], ThreadExchange(hub, r), x[t0:t0 + Ts[r]], ys[r], biases[r], alpha,
                                         T_total=T)
            torch.cuda.synchronize()
        except BaseException as e:  # noqa: BLE001 - reported below
            errors[r] = e
            hub.bar.abort()

    th = [threading.Thread(target=run, args=(r,)) for r in range(G)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert all(e is None for e in errors), errors
    # reference 1: the single-GPU layer on each rank's tokens, all experts local
    for r in range(G):
        t0 = sum(Ts[:r])
        dims = abi.Dims(Ts[r], dm, df, E, K, cf)
        ws = abi.alloc_workspace(dims)
        y1 = torch.empty(Ts[r], dm, dtype=torch.float32, device=d)
        idx = torch.empty(Ts[r], K, dtype=torch.int32, device=d)
        abi.moe_layer_forward(dims, x[t0:t0 + Ts[r]].contiguous(), Wr, bias0.clone(), 0.0, W13p, W2p, y1, ws,
                              {"topk_idx": idx})
        torch.cuda.synchronize()
        assert torch.equal(idx, steps[r].idx)   # same router kernels, same routing
        assert rel_l2(f64(ys[r]), f64(y1)) <= 1e-5
        # reference 2: the fp64 oracle on the rank's tokens
        ref = O.moe_layer(f64(x[t0:t0 + Ts[r]]), f64(Wr), f64(W1), f64(W3), f64(W2), K, cf,
                          bias32=bias0.cpu().numpy())
        unc = uncertain_tokens(idx.cpu().numpy(), ref["idx"], E, ref["capacity"])
        assert unc.mean() <= 0.05
        keep = ~unc
        assert_close_y(f64(ys[r])[keep], ref["y"][keep], Y_MAX_ABS, Y_REL_L2, f"rank {r} y")
    # every rank applied the same bias update, from the counts of all ranks' tokens
    for r in range(1, G):
        assert torch.equal(biases[r], biases[0]) and torch.equal(totals[r], totals[0])
    assert int(totals[0].sum().item()) == T * K
