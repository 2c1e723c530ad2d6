"""Expert parallelism on CPU ranks: the step sequence, the split plan and the
exchanges of moe_layer_gemm_b200.ep over gloo, world sizes 2 and 4.

Each rank runs ep_forward with the real DistExchange (all_to_all_single and
all_reduce over gloo) and local steps taken from the oracle (fp64), so what
is checked is the host-side plan: which rows go where, the regroup by local
expert, the return path and the combine.  Expected values: the oracle's
single-process layer on each rank's own tokens (routing and capacity are per
rank), and the bias update from the counts of all ranks' tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from moe_layer_gemm_b200 import ep, synth
from oracle import moe_oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleSteps:
    """The local steps from the oracle's functions, on torch CPU tensors."""

    out_dtype = torch.float64

    def __init__(self, x64, Wr64, W1, W3, W2, K, cf, rank, n_ranks):
        self.x64, self.Wr64 = x64, Wr64
        self.E = Wr64.shape[1]
        self.K, self.cf = K, cf
        self.rank, self.n_ranks = rank, n_ranks
        blk = ep.expert_block(rank, n_ranks, self.E)
        self.E_local = len(blk)
        self.W1, self.W3, self.W2 = W1[blk.start:blk.stop], W3[blk.start:blk.stop], W2[blk.start:blk.stop]

    def route(self, x, bias):
        l32 = O.router_logits(self.x64, self.Wr64).astype(np.float32)
        b = None if bias is None else bias.numpy()
        idx, w, _ = O.route_from_logits_f32(l32, self.K, b)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w)

    def dispatch(self, idx, x):
        T = self.x64.shape[0]
        dsp = O.dispatch(idx.numpy(), self.E, O.capacity(T, self.K, self.E, self.cf))
        x_perm = torch.from_numpy(self.x64[dsp["src"]].copy())
        return (torch.from_numpy(dsp["counts"].astype(np.int32)), torch.from_numpy(dsp["kept"].astype(np.int32)),
                torch.from_numpy(dsp["offsets"].astype(np.int32)), torch.from_numpy(dsp["inv"].astype(np.int32)),
                x_perm)

    def local_experts(self, recv_counts, rows):
        rc = recv_counts.numpy().reshape(self.n_ranks, self.E_local)
        ids = np.concatenate([np.repeat(np.arange(self.E_local), rc[s]) for s in range(self.n_ranks)])
        g = O.dispatch(ids[:, None], self.E_local)          # stable grouping by local expert
        row_of = g["inv"][:, 0]
        R = rows.numpy()
        grouped = np.empty_like(R)
        grouped[row_of] = R
        Y = np.empty_like(R)
        off = g["offsets"]
        for e in range(self.E_local):
            if off[e + 1] > off[e]:
                Y[off[e]:off[e + 1]] = O.swiglu_ffn(grouped[off[e]:off[e + 1]], self.W1[e], self.W3[e], self.W2[e])
        return torch.from_numpy(Y[row_of])

    def combine(self, y_back, inv, w, y):
        y[:] = torch.from_numpy(O.combine(y_back.numpy(), inv.numpy(), w.numpy(), y.shape[0]))

    def bias_update(self, counts_total, T_total, alpha, bias):
        bias[:] = torch.from_numpy(O.bias_update(bias.numpy(), counts_total.numpy(), T_total, self.K, alpha))


def _inputs(seed, Ts, d, f, E, hot):
    T = sum(Ts)
    x = synth.normal_bf16((T, d), seed, synth.STREAM_X).double().numpy()
    Wr = synth.normal_bf16((d, E), seed, synth.STREAM_WR, 0.2).double().numpy()
    W1 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W1, 0.05).double().numpy()
    W3 = synth.normal_bf16((E, d, f), seed, synth.STREAM_W3, 0.05).double().numpy()
    W2 = synth.normal_bf16((E, f, d), seed, synth.STREAM_W2, 0.05).double().numpy()
    bias = np.zeros(E, np.float32)
    bias[hot] = 50.0          # these experts take every token's first slots
    return x, Wr, W1, W3, W2, bias


def _rank(rank, world, port, case, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Ts, d, f, E, K, cf, hot, alpha = case
        x, Wr, W1, W3, W2, bias0 = _inputs(7, Ts, d, f, E, hot)
        t0 = sum(Ts[:rank])
        xr = x[t0:t0 + Ts[rank]]
        steps = OracleSteps(xr, Wr, W1, W3, W2, K, cf, rank, world)
        xchg = ep.DistExchange()
        y = torch.full((Ts[rank], d), float("nan"), dtype=torch.float64)
        bias = torch.from_numpy(bias0.copy())
        counts, total = ep.ep_forward(steps, xchg, torch.from_numpy(xr), y, bias, alpha, T_total=sum(Ts))
        ref = O.moe_layer(xr, Wr, W1, W3, W2, K, cf, bias32=bias0)
        err = float(np.max(np.abs(y.numpy() - ref["y"]))) if Ts[rank] else 0.0
        scale = float(np.max(np.abs(ref["y"]))) if Ts[rank] else 1.0
        # the bias update uses every rank's counts
        idx_all, _, _ = O.route_from_logits_f32(O.router_logits(x, Wr).astype(np.float32), K, bias0)
        cnt_all = O.expert_counts(idx_all, E)
        b_ref = O.bias_update(bias0, cnt_all, sum(Ts), K, alpha)
        out[rank] = (err / max(scale, 1e-300), bool(np.array_equal(counts.numpy(), ref["counts"])),
                     bool(np.array_equal(bias.numpy().view(np.uint32), b_ref.view(np.uint32))),
                     bool(np.array_equal(total.numpy(), cnt_all)) if total is not None else True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


CASES = {
    # ranks with different batch sizes, no capacity, bias update
    "two_ranks": ([37, 52], 64, 96, 8, 2, 0.0, [], 1e-3),
    # four ranks, capacity per rank's batch, one rank's experts hot
    "four_ranks_capacity": ([30, 41, 16, 57], 64, 96, 8, 2, 1.0, [1], 1e-3),
    # four ranks, every token's slots on experts 0 and 1 (rank 0's): ranks 1-3 receive no rows
    "four_ranks_all_to_one": ([20, 33, 8, 25], 32, 64, 8, 2, 0.0, [0, 1], 0.0),
    # a rank with no tokens at all
    "empty_rank": ([40, 0, 23, 31], 32, 64, 8, 2, 0.0, [], 1e-3),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_ep_forward_matches_oracle_per_rank(name):
    case = CASES[name]
    world = len(case[0])
    out = mp.get_context("spawn").Manager().list([None] * world)
    mp.spawn(_rank, args=(world, _free_port(), case, out), nprocs=world, join=True)
    for r in range(world):
        rel, counts_ok, bias_ok, total_ok = out[r]
        assert rel <= 1e-12, (r, rel)
        assert counts_ok and bias_ok and total_ok, (r, out[r])


def test_plan_helpers():
    assert list(ep.expert_block(2, 4, 256)) == list(range(128, 192))
    with pytest.raises(ValueError):
        ep.expert_block(0, 3, 8)
    offsets = [0, 3, 3, 7, 10, 10, 12, 20, 21]     # E = 8 over 4 ranks: blocks of 2 experts
    assert ep.send_splits(offsets, 4, 2) == [3, 7, 2, 9]
    assert sum(ep.send_splits(offsets, 4, 2)) == offsets[-1]
    assert ep.recv_splits([1, 2, 0, 0, 5, 1, 3, 3], 4, 2) == [3, 0, 6, 6]
