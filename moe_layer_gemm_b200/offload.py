"""Expert offloading: experts kept in host memory as group-wise INT4, an LRU
cache of experts in GPU memory, and prefetching predicted from the routing
history.

"MoE inference engineering in practice" (ybb.press/quantum-computing/18594),
section 3.2: when the experts do not all fit in GPU memory (its example is
DeepSeek-V3's 256 routed experts), offload some to CPU memory; keep an LRU
cache of the frequently used experts on the GPU; predict from the routing
history which experts the next batch needs and load them ahead of time; store
the offloaded experts group-wise quantized to INT4 to cut the transfer volume.

One step of OffloadedLayer (the main stream; a copy stream and an unpack
stream for the experts that miss; a side stream for the prefetch):
  1 route and dispatch the batch (moe_route, moe_permute)
  2 read the per-expert kept counts on the host: the step's one host
    synchronisation, since which experts to load is decided here
  3 the cache plan (ExpertCache): hits refresh their slot; each miss, in
    ascending expert order, takes the least recently used slot holding no
    expert this step needs (equal last use: the lower slot)
  4 each missed expert's INT4 codes are copied from page-locked host memory
    into a device staging buffer by the copy engine (the host link's full
    rate, no SM time), and expanded into its slot (moe_int4_unpack) as soon
    as its copy has landed
  5 meanwhile the expert GEMMs of the resident experts run
    (moe_expert_ffn_slots with the missed experts skipped); then those of
    the missed experts (the complementary table), then the combine
  6 update the prediction (HistoryPredictor: a per-expert fp32 moving average
    of routed counts) and expand the predicted experts that are not resident,
    on the side stream, into slots holding no expert of this step; the next
    step waits for it before touching the cache

The cache bookkeeping is host control logic; every data movement and every
computation runs in the library's kernels.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np
import torch

from . import abi


class ExpertCache:
    """Which expert sits in which of n_slots cache slots, least recently used
    first out (see the module notes for the exact rule)."""

    def __init__(self, n_slots: int):
        if n_slots < 1:
            raise ValueError("the cache needs at least one slot")
        self.n_slots = n_slots
        self.expert_in = [-1] * n_slots   # expert held by each slot
        self.used_at = [-1] * n_slots     # step of the slot's last use (-1: never)
        self.where: Dict[int, int] = {}   # expert -> slot
        self.from_prefetch = set()        # experts the last prefetch loaded
        self.step = -1

    def _victim(self, keep) -> int:
        best = None
        for sl in range(self.n_slots):
            if self.expert_in[sl] in keep:
                continue
            key = (self.used_at[sl], sl)
            if best is None or key < best:
                best = key
        return -1 if best is None else best[1]

    def _place(self, e: int, sl: int):
        old = self.expert_in[sl]
        if old >= 0:
            self.where.pop(old, None)
        self.expert_in[sl] = e
        self.where[e] = sl
        self.used_at[sl] = self.step

    def plan(self, needed: Sequence[int]):
        """Demand plan of the next step: (hits, prefetch_hits, misses, loads)."""
        self.step += 1
        need = sorted({int(e) for e in needed})
        if len(need) > self.n_slots:
            raise RuntimeError(f"{len(need)} experts needed at once, the cache has {self.n_slots} slots")
        keep = set(need)
        hits, phits, misses, loads = [], [], [], []
        for e in need:
            if e in self.where:
                (phits if e in self.from_prefetch else hits).append(e)
                self.used_at[self.where[e]] = self.step
            else:
                misses.append(e)
        for e in misses:
            sl = self._victim(keep)
            self._place(e, sl)
            loads.append((e, sl))
        self.from_prefetch = set()
        self._keep = keep
        return hits, phits, misses, loads

    def plan_prefetch(self, predicted: Sequence[int]) -> List[Tuple[int, int]]:
        """Load plan for predicted experts after this step (slots of this
        step's experts are kept)."""
        loads = []
        for e in predicted:
            e = int(e)
            if e in self.where:
                continue
            sl = self._victim(self._keep)
            if sl < 0:
                break
            self._place(e, sl)
            self.from_prefetch.add(e)
            loads.append((e, sl))
        return loads

    def slot_table(self, E: int) -> np.ndarray:
        t = np.full(E, -1, dtype=np.int32)
        for e, sl in self.where.items():
            t[e] = sl
        return t


class HistoryPredictor:
    """Experts likely needed next: a per-expert moving average of routed
    counts, c <- fl32(fl32(beta c) + n) in fp32; the `width` largest (equal
    values: lower expert first)."""

    def __init__(self, E: int, width: int, beta: float = 0.75):
        self.c = None
        self.beta = np.float32(beta)
        self.width = width
        self.E = E

    def update(self, counts) -> List[int]:
        n = np.asarray(counts, dtype=np.float32)
        self.c = n.copy() if self.c is None else (self.beta * self.c + n).astype(np.float32)
        # stable descending order: equal averages keep the lower expert first
        order = sorted(range(self.E), key=lambda e: (-float(self.c[e]), e))
        return order[: self.width]


def quantize_experts_to_host(dims, W1, W3, W2, stream=None):
    """INT4 codes and scales of all experts (moe_int4_pack on the device), in
    page-locked host memory: (q13, s13, q2, s2)."""
    n13, ns13, n2, ns2 = abi.moe_int4_bytes(dims)
    dev = W1.device
    q13 = torch.empty(n13, dtype=torch.uint8, device=dev)
    s13 = torch.empty(ns13 // 4, dtype=torch.float32, device=dev)
    q2 = torch.empty(n2, dtype=torch.uint8, device=dev)
    s2 = torch.empty(ns2 // 4, dtype=torch.float32, device=dev)
    abi.moe_int4_pack(dims, W1, W3, W2, q13, s13, q2, s2, stream)
    host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (q13, s13, q2, s2)]
    for h, t in zip(host, (q13, s13, q2, s2)):
        h.copy_(t)
    return tuple(host)


class OffloadedLayer:
    """The MoE layer with its experts in host memory (INT4) and n_slots of
    them cached on the GPU.

    dims      the batch shape (T tokens per step, all E experts)
    Wr        [d, E] bf16 router weight on the device
    q13..s2   INT4 codes and scales of all experts in page-locked host memory
    n_slots   experts the GPU cache holds (at least the experts one step needs)
    prefetch  experts predicted and loaded ahead after each step (0: none)
    """

    def __init__(self, dims: abi.Dims, Wr, q13, s13, q2, s2, n_slots: int, prefetch: int = 0):
        self.dims = dims
        self.Wr = Wr
        self.dev = Wr.device
        self.q13, self.s13, self.q2, self.s2 = q13, s13, q2, s2
        self.n_slots = n_slots
        per13, per2 = (b // dims.E for b in abi.moe_packed_weight_bytes(dims))
        self.W13c = torch.empty(n_slots * per13 // 2, dtype=torch.bfloat16, device=self.dev)
        self.W2c = torch.empty(n_slots * per2 // 2, dtype=torch.bfloat16, device=self.dev)
        n13, ns13, n2, ns2 = abi.moe_int4_bytes(dims)
        self.bytes_per_expert = (n13 + ns13 + n2 + ns2) // dims.E
        self.cache = ExpertCache(n_slots)
        self.predictor = HistoryPredictor(dims.E, prefetch) if prefetch > 0 else None
        T, K, E, d, f = dims.T, dims.K, dims.E, dims.d_model, dims.d_ff
        i32 = dict(dtype=torch.int32, device=self.dev)
        self.ws = abi.alloc_workspace(dims, self.dev)
        self.idx, self.w = torch.empty(T, K, **i32), torch.empty(T, K, dtype=torch.float32, device=self.dev)
        self.counts, self.kept = torch.empty(E, **i32), torch.empty(E, **i32)
        self.offsets, self.inv = torch.empty(E + 1, **i32), torch.empty(T, K, **i32)
        self.src, self.nd = torch.empty(T * K, **i32), torch.empty(1, **i32)
        self.x_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=self.dev)
        self.h = torch.empty(T * K, f, dtype=torch.bfloat16, device=self.dev)
        self.y_perm = torch.empty(T * K, d, dtype=torch.float32, device=self.dev)
        # slot tables: [0] the resident experts (misses skipped), [1] the misses
        self.slot_dev = [torch.full((E,), abi.MOE_SLOT_SKIP, **i32) for _ in range(2)]
        self.slot_host = [torch.empty(E, dtype=torch.int32, pin_memory=True) for _ in range(2)]
        self.counts_host = torch.empty(2 * E, dtype=torch.int32, pin_memory=True)
        self.side = torch.cuda.Stream(self.dev)
        self.copy = torch.cuda.Stream(self.dev)
        self.unpack_stream = torch.cuda.Stream(self.dev)
        self.dispatched = torch.cuda.Event()
        self.unpacked = torch.cuda.Event()
        # per-expert views of the host codes, and device staging buffers for the misses
        self.host_views = tuple(t.view(E, -1) for t in (q13, s13, q2, s2))
        self.stage = None
        self.log: List[dict] = []

    def _unpack(self, loads, stream):
        """Expand experts straight from page-locked host memory (the prefetch)."""
        if loads:
            abi.moe_int4_unpack(self.dims, [e for e, _ in loads], [s for _, s in loads], self.q13, self.s13,
                                self.q2, self.s2, self.n_slots, self.W13c, self.W2c, stream)

    def _stage(self, n: int):
        """Device staging buffers for n missed experts (grown on need)."""
        if self.stage is None or self.stage[0].shape[0] < n:
            self.stage = tuple(torch.empty((n, v.shape[1]), dtype=v.dtype, device=self.dev) for v in self.host_views)
            for t in self.stage:  # used on the copy and unpack streams: the allocator must wait for them
                t.record_stream(self.copy)
                t.record_stream(self.unpack_stream)
        return self.stage

    def _load_misses(self, loads):
        """Copy each missed expert's codes to the device on the copy stream and
        expand it into its slot on the unpack stream once its copy has landed;
        self.unpacked marks the end."""
        stage = self._stage(len(loads))
        unpack = self.unpack_stream
        for j, (e, sl) in enumerate(loads):
            copied = torch.cuda.Event()
            with torch.cuda.stream(self.copy):
                for dst, src in zip(stage, self.host_views):
                    dst[j].copy_(src[e], non_blocking=True)
                copied.record(self.copy)
            unpack.wait_event(copied)
            flat = tuple(t.view(-1) for t in stage)
            abi.moe_int4_unpack(self.dims, [j], [sl], *flat, self.n_slots, self.W13c, self.W2c, unpack)
        self.unpacked.record(unpack)

    def _ffn(self, table: int, which: np.ndarray):
        """Expert GEMMs of the experts with which[e] set (the others skipped)."""
        dims = self.dims
        slots = self.cache.slot_table(dims.E)
        t = np.where(which, slots, abi.MOE_SLOT_SKIP).astype(np.int32)
        self.slot_host[table].copy_(torch.from_numpy(t))
        self.slot_dev[table].copy_(self.slot_host[table], non_blocking=True)
        abi.moe_expert_ffn_slots(dims, self.x_perm, self.offsets, self.slot_dev[table], self.n_slots, self.W13c,
                                 self.W2c, self.h, self.y_perm, self.ws)

    def forward(self, x, y):
        dims, E = self.dims, self.dims.E
        main = torch.cuda.current_stream(self.dev)
        abi.moe_route(dims, x, self.Wr, None, None, self.idx, self.w, None, self.ws)
        abi.moe_permute(dims, self.idx, x, self.counts, self.kept, self.offsets, self.inv, self.src, self.x_perm,
                        self.nd, self.ws)
        self.dispatched.record(main)
        self.counts_host[:E].copy_(self.counts, non_blocking=True)
        self.counts_host[E:].copy_(self.kept, non_blocking=True)
        main.synchronize()                                   # the step's one host synchronisation
        counts = self.counts_host[:E].numpy().copy()
        kept = self.counts_host[E:].numpy()
        needed = [int(e) for e in np.nonzero(kept)[0]]
        hits, phits, misses, loads = self.cache.plan(needed)
        main.wait_stream(self.side)                           # the last prefetch has landed
        missed = np.zeros(E, dtype=bool)
        missed[misses] = True
        resident = (kept > 0) & ~missed
        if loads:
            # the copies start after the prefetch (its slots) and the last step's reads of the slots
            self.copy.wait_stream(main)
            self.unpack_stream.wait_stream(main)
            self._load_misses(loads)
        if resident.any():
            self._ffn(0, resident)                            # overlaps the copies of the misses
        if loads:
            main.wait_event(self.unpacked)
            self._ffn(1, missed)
        abi.moe_combine(dims, self.y_perm, self.inv, self.w, y)
        ploads = []
        if self.predictor is not None:
            predicted = self.predictor.update(counts)
            ploads = self.cache.plan_prefetch(predicted)
            if ploads:
                # slots of this step's experts are kept, and the slots written
                # here were last read by an earlier step's GEMMs, which precede
                # this step's dispatch on the main stream: the prefetch overlaps
                # this step's GEMMs and combine
                self.side.wait_event(self.dispatched)
                self._unpack(ploads, self.side)
        rec = dict(needed=needed, hits=hits, prefetch_hits=phits, misses=misses, loads=loads, prefetch_loads=ploads,
                   unpacked_bytes=(len(loads) + len(ploads)) * self.bytes_per_expert)
        self.log.append(rec)
        return rec
