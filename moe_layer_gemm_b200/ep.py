"""Expert-parallel MoE layer: the experts spread over G GPUs, one process each.

"MoE computation notes" (cf-1.com/news/5905749), section 4.2, and "MoE
inference engineering in practice" (ybb.press/quantum-computing/18594),
section 2.2: expert parallelism places different experts on different GPUs;
each GPU routes its own tokens, an all-to-all sends every token row to the
GPU that holds its expert, each GPU runs its local experts, and a second
all-to-all brings the results back for the weighted combine.

Partition: E experts over G ranks in contiguous blocks; rank r holds experts
r E_l .. (r + 1) E_l - 1 (E_l = E / G) and only their packed weights.  Each
rank routes and dispatches its own batch, so a capacity limit applies to each
rank's batch, and every rank's output equals the single-GPU layer's output on
its own tokens.  The aux-free bias update uses the counts summed over ranks
and the total token count, so every rank applies the same update.

One step, for rank r:
  1 route (moe_route) and dispatch (moe_permute) the rank's tokens over all E
    experts; dispatch rows are expert-major, so the rows bound for rank j are
    the contiguous block offsets[j E_l] .. offsets[(j + 1) E_l]
  2 exchange the per-(destination, local expert) row counts (all-to-all)
  3 exchange the rows (all-to-all; splits from the counts)
  4 regroup the received rows by local expert (moe_ep_regroup)
  5 run the local experts (moe_expert_ffn)
  6 put the results back in the received order (moe_combine, K = 1, unit
    weights: an exact copy)
  7 return the rows to their source ranks (all-to-all, splits swapped)
  8 combine (moe_combine) with the step-1 inverse map and weights
  9 optionally, the bias update from the counts summed over ranks

Every step that computes runs in the library's CUDA kernels (CudaSteps); this
module orders the calls and hands buffers to the exchange, which moves them
between ranks (DistExchange: torch.distributed all_to_all_single, NCCL on
GPUs).  The step sequence (ep_forward) is written against two small
interfaces, the steps and the exchange, so the host-side plan can be checked
on CPU ranks as well.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import abi


# ---------------------------------------------------------------- the plan

def expert_block(rank: int, n_ranks: int, E: int) -> range:
    """Experts held by `rank`: a contiguous block of E / n_ranks."""
    if E % n_ranks != 0:
        raise ValueError(f"E = {E} experts do not split evenly over {n_ranks} ranks")
    El = E // n_ranks
    return range(rank * El, (rank + 1) * El)


def send_splits(offsets: Sequence[int], n_ranks: int, E_local: int) -> List[int]:
    """Rows bound for each destination rank: the dispatch offsets' blocks."""
    return [int(offsets[(j + 1) * E_local]) - int(offsets[j * E_local]) for j in range(n_ranks)]


def recv_splits(recv_counts: Sequence[int], n_ranks: int, E_local: int) -> List[int]:
    """Rows arriving from each source rank: its counts for the local experts."""
    return [int(sum(int(c) for c in recv_counts[s * E_local:(s + 1) * E_local])) for s in range(n_ranks)]


# ---------------------------------------------------------------- exchange

class DistExchange:
    """The two all-to-all exchanges and the count sum over torch.distributed
    (NCCL between GPUs).  bf16 rows travel as their 16-bit patterns."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.n_ranks = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def counts(self, send: torch.Tensor) -> torch.Tensor:
        """send [n_ranks * E_l]: block j for rank j -> recv block s from rank s."""
        out = torch.empty_like(send)
        self.dist.all_to_all_single(out, send, group=self.group)
        return out

    def rows(self, send: torch.Tensor, splits_out: List[int], splits_in: List[int]) -> torch.Tensor:
        wire = send.view(torch.int16) if send.dtype == torch.bfloat16 else send
        out = wire.new_empty((sum(splits_in),) + tuple(send.shape[1:]))
        self.dist.all_to_all_single(out, wire.contiguous(), splits_in, splits_out, group=self.group)
        return out.view(send.dtype)

    def sum(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, group=self.group)
        return t


# ---------------------------------------------------------------- local steps

class CudaSteps:
    """Each local step of the expert-parallel layer in the library's kernels.

    dims      the rank's batch: T its tokens, E the global expert count
    Wr        [d, E] bf16 router weight (every rank holds all of it)
    W13p, W2p packed weights of this rank's E / n_ranks experts only
    """

    out_dtype = torch.float32  # rows the local experts return (fp32 accumulations)

    def __init__(self, dims: abi.Dims, rank: int, n_ranks: int, Wr, W13p, W2p):
        self.dims = dims
        self.rank, self.n_ranks = rank, n_ranks
        self.E_local = len(expert_block(rank, n_ranks, dims.E))
        self.Wr, self.W13p, self.W2p = Wr, W13p, W2p
        self.dev = Wr.device
        self.ws = abi.alloc_workspace(dims, self.dev)
        T, K, E, d = dims.T, dims.K, dims.E, dims.d_model
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.idx = torch.empty(T, K, **i32)
        self.w = torch.empty(T, K, dtype=torch.float32, device=self.dev)
        self.counts = torch.empty(E, **i32)
        self.kept = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.inv = torch.empty(T, K, **i32)
        self.src = torch.empty(T * K, **i32)
        self.x_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=self.dev)
        self.n_dropped = torch.empty(1, **i32)
        self._local_ws = {}

    def route(self, x, bias):
        abi.moe_route(self.dims, x, self.Wr, bias, None, self.idx, self.w, None, self.ws)
        return self.idx, self.w

    def dispatch(self, idx, x):
        abi.moe_permute(self.dims, idx, x, self.counts, self.kept, self.offsets, self.inv, self.src, self.x_perm,
                        self.n_dropped, self.ws)
        return self.counts, self.kept, self.offsets, self.inv, self.x_perm

    def _local(self, n):
        """Buffers of the local expert step for n received rows: grown to the
        next power of two rows when too small, kept for reuse."""
        b = self._local_ws
        d, f = self.dims.d_model, self.dims.d_ff
        need_ws = abi.moe_workspace_size(abi.Dims(n, d, f, self.E_local, 1))
        if b.get("cap", 0) < n:
            cap = 1 << max(0, (n - 1).bit_length())
            b.update(cap=cap,
                     rows=torch.empty(cap, d, dtype=torch.bfloat16, device=self.dev),
                     h=torch.empty(cap, f, dtype=torch.bfloat16, device=self.dev),
                     y=torch.empty(cap, d, dtype=torch.float32, device=self.dev),
                     back=torch.empty(cap, d, dtype=torch.float32, device=self.dev),
                     row_of=torch.empty(cap, dtype=torch.int32, device=self.dev),
                     ones=torch.ones(cap, dtype=torch.float32, device=self.dev),
                     offsets=torch.empty(self.E_local + 1, dtype=torch.int32, device=self.dev))
        if b.get("ws") is None or b["ws"].numel() < need_ws:
            b["ws"] = torch.zeros(need_ws, dtype=torch.uint8, device=self.dev)
        return b

    def local_experts(self, recv_counts, rows):
        """Steps 4-6: regroup, run the local experts, restore the received
        order (a unit-weight, one-slot combine: an exact copy, up to the sign
        of a zero)."""
        n = rows.shape[0]
        b = self._local(n)
        d = self.dims.d_model
        rows_g, row_of, off = b["rows"][:n], b["row_of"][:n], b["offsets"]
        abi.moe_ep_regroup(self.n_ranks, self.E_local, recv_counts, rows, rows_g, off, row_of)
        dl = abi.Dims(n, d, self.dims.d_ff, self.E_local, 1)
        y_g = b["y"][:n]
        abi.moe_expert_ffn(dl, rows_g, off, self.W13p, self.W2p, b["h"][:n], y_g, b["ws"])
        back = b["back"][:n]
        abi.moe_combine(dl, y_g, row_of.view(n, 1), b["ones"][:n].view(n, 1), back)
        return back

    def combine(self, y_back, inv, w, y):
        abi.moe_combine(self.dims, y_back, inv, w, y)

    def bias_update(self, counts_total, T_total: int, alpha: float, bias):
        dg = abi.Dims(T_total, self.dims.d_model, self.dims.d_ff, self.dims.E, self.dims.K)
        abi.moe_bias_update(dg, counts_total, alpha, bias)


def ep_forward(steps, xchg, x, y, bias=None, alpha: float = 0.0, T_total: Optional[int] = None):
    """One expert-parallel layer step for this rank (see the module notes).

    steps  the local steps (CudaSteps on GPUs)
    xchg   the exchange (DistExchange)
    x, y   this rank's tokens and output rows
    bias   [E] fp32, the same on every rank; with alpha != 0 it is updated in
           place from the counts summed over ranks (T_total = all ranks'
           tokens), after this step's routing
    Returns this rank's per-expert counts (before drops) and, with a bias
    update, the counts summed over ranks.
    """
    G, El = steps.n_ranks, steps.E_local
    idx, w = steps.route(x, bias)
    counts, kept, offsets, inv, x_perm = steps.dispatch(idx, x)
    recv_counts = xchg.counts(kept)
    # the row exchange needs its sizes on the host: E + 1 and n_ranks * E_l integers
    off_h = offsets.tolist()
    rc_h = recv_counts.tolist()
    s_out = send_splits(off_h, G, El)
    s_in = recv_splits(rc_h, G, El)
    rows = xchg.rows(x_perm[: sum(s_out)], s_out, s_in)
    if sum(s_in) > 0:
        back = steps.local_experts(recv_counts, rows)
    else:  # nothing received: still part of the return exchange
        back = torch.empty((0,) + tuple(y.shape[1:]), dtype=steps.out_dtype, device=y.device)
    y_perm = xchg.rows(back, s_in, s_out)
    if y_perm.shape[0] == 0:  # every slot dropped: the combine reads no row but wants a buffer
        y_perm = torch.zeros((1,) + tuple(y.shape[1:]), dtype=steps.out_dtype, device=y.device)
    steps.combine(y_perm, inv, w, y)
    total = None
    if bias is not None and alpha != 0.0:
        total = xchg.sum(counts.clone())
        steps.bias_update(total, int(T_total), alpha, bias)
    return counts, total
