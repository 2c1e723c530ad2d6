"""Seeded, index-addressable synthetic inputs for the MoE layer.

This module only draws numbers: it holds none of the layer's arithmetic (no
routing, no softmax, no expert math).  Both the CUDA library's callers and the
CPU oracle's callers take their inputs from here, so the two sides always see
the same bits.

Generator
---------
Element ``i`` of stream ``(seed, stream_id)`` is

    h  = lowbias32(lo32(i) XOR k_hi)         k_hi = lowbias32(hi32(i) XOR key)
    z  = Q[h >> 12]                           (a 2**20-entry quantile table)
    v  = bf16_rne(fp32(z) * fp32(std))

where ``Q[j]`` is the standard-normal quantile at ``(j + 0.5) / 2**20``
(inverse-transform sampling; the table is computed once on the host in fp64 and
rounded to fp32).  ``lowbias32`` is Chris Wellons' published 32-bit integer
hash.  Every step is exact integer arithmetic, one table gather, one correctly
rounded fp32 multiply and one round-to-nearest-even conversion, so the result is
bit-identical on the CPU and on a GPU: large tensors can be generated on the
device and any slice regenerated on the host.

The tails are truncated at the table's ends (about +-4.9 sigma), which changes
the variance by less than 1e-5 relative.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field
from typing import Optional

import torch

_M32 = 0xFFFFFFFF
_TABLE_BITS = 20
_TABLE_CACHE: dict = {}

# Stream identifiers: one independent stream per tensor role.
STREAM_X = 1
STREAM_WR = 2
STREAM_W1 = 3
STREAM_W3 = 4
STREAM_W2 = 5
STREAM_LOGITS = 6
STREAM_IDX = 7
STREAM_MISC = 8
STREAM_SKEW = 9


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2**32 for 0 <= x < 2**32, without int64 overflow."""
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def _lowbias32(x: torch.Tensor) -> torch.Tensor:
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _lowbias32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & _M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & _M32
    x ^= x >> 16
    return x


def stream_key(seed: int, stream: int) -> int:
    """32-bit key of stream ``stream`` under ``seed``."""
    k = _lowbias32_int(seed * 0x9E3779B9 + 0x632BE5AB)
    return _lowbias32_int(k ^ (stream * 0x85EBCA77 + 0x27D4EB2F))


def _quantile_table(device) -> torch.Tensor:
    dev = torch.device(device)
    key = (dev.type, dev.index)
    t = _TABLE_CACHE.get(key)
    if t is None:
        n = 1 << _TABLE_BITS
        p = (torch.arange(n, dtype=torch.float64) + 0.5) / n
        host = torch.special.ndtri(p).to(torch.float32)
        t = host.to(dev)
        _TABLE_CACHE[key] = t
    return t


def hash_u32(n: int, seed: int, stream: int, device="cpu", offset: int = 0) -> torch.Tensor:
    """n uniform 32-bit integers (as int64) of elements offset..offset+n-1."""
    key = stream_key(seed, stream)
    out = torch.empty(n, dtype=torch.int64, device=device)
    pos = 0
    while pos < n:
        i0 = offset + pos
        hi = i0 >> 32
        # stay inside one 2**32 block so k_hi is a scalar
        take = min(n - pos, ((hi + 1) << 32) - i0)
        khi = _lowbias32_int(hi ^ key)
        lo = torch.arange(i0 & _M32, (i0 & _M32) + take, dtype=torch.int64, device=device)
        out[pos:pos + take] = _lowbias32(lo ^ khi)
        pos += take
    return out


def normal_f32(n: int, seed: int, stream: int, device="cpu", offset: int = 0) -> torch.Tensor:
    """n standard-normal fp32 draws of elements offset..offset+n-1."""
    h = hash_u32(n, seed, stream, device, offset)
    return _quantile_table(device)[h >> (32 - _TABLE_BITS)]


def normal_bf16(shape, seed: int, stream: int, std: float = 1.0, device="cpu",
                chunk: int = 1 << 24, col_scale: Optional[torch.Tensor] = None,
                col_shift: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16 tensor of N(0, std^2) draws, row-major element order.

    ``col_scale`` / ``col_shift`` (fp32, one value per last-dim column) give
    v = bf16(fp32(fp32(z*std) * scale) + shift) and are used to shape router
    weights; both are exact-rounded fp32 operations, so device independent.
    """
    shape = tuple(int(s) for s in shape)
    numel = 1
    for s in shape:
        numel *= s
    out = torch.empty(numel, dtype=torch.bfloat16, device=device)
    ncol = shape[-1] if shape else 1
    std32 = torch.tensor(std, dtype=torch.float32, device=device)
    if col_scale is not None:
        col_scale = col_scale.to(device=device, dtype=torch.float32)
    if col_shift is not None:
        col_shift = col_shift.to(device=device, dtype=torch.float32)
    pos = 0
    while pos < numel:
        take = min(chunk, numel - pos)
        v = normal_f32(take, seed, stream, device, pos) * std32
        if col_scale is not None or col_shift is not None:
            cols = torch.arange(pos, pos + take, device=device) % ncol
            if col_scale is not None:
                v = v * col_scale[cols]
            if col_shift is not None:
                v = v + col_shift[cols]
        out[pos:pos + take] = v.to(torch.bfloat16)
        pos += take
    return out.view(shape)


def distinct_choices(T: int, E: int, K: int, seed: int, stream: int = STREAM_IDX,
                     device="cpu", weights: Optional[torch.Tensor] = None) -> torch.Tensor:
    """[T, K] int32: for each row, K distinct values in [0, E) in random order.

    Draws one random key per (row, value) and keeps the K smallest keys (a
    random permutation prefix).  ``weights`` (length E, positive) skews the
    choice: key = u ** (1/w) keeps larger w more often (weighted sampling
    without replacement).
    """
    u = hash_u32(T * E, seed, stream, device).view(T, E).to(torch.float64)
    u = (u + 0.5) / 4294967296.0
    if weights is not None:
        w = weights.to(device=device, dtype=torch.float64)
        key = -torch.log(u) / w
    else:
        key = u
    order = torch.argsort(key, dim=1, stable=True)
    return order[:, :K].to(torch.int32).contiguous()


def logits_f32(T: int, E: int, seed: int, std: float = 1.0, device="cpu",
               tie_frac: float = 0.0) -> torch.Tensor:
    """[T, E] fp32 synthetic router logits.

    With ``tie_frac`` > 0 that fraction of rows is rounded to a coarse grid
    (multiples of 0.25) so exact ties occur, and zeros carry random signs
    (+0.0 / -0.0), to exercise the tie rule.
    """
    v = normal_f32(T * E, seed, STREAM_LOGITS, device).view(T, E) * std
    if tie_frac > 0:
        sel = hash_u32(T, seed, STREAM_MISC, device) < int(tie_frac * 4294967296.0)
        coarse = torch.round(v * 4.0) / 4.0
        sgn = (hash_u32(T * E, seed + 1, STREAM_MISC, device).view(T, E) & 1).bool()
        coarse = torch.where((coarse == 0) & sgn, torch.full_like(coarse, -0.0), coarse)
        v = torch.where(sel[:, None], coarse, v)
    return v.to(torch.float32).contiguous()


# --------------------------------------------------------------------------
# Workloads: the five layer configurations with their input recipes.
# --------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    K: int
    capacity_factor: float = 0.0
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    use_bias: bool = False
    alpha: float = 0.0
    steps: int = 1
    skew: str = "none"             # none | col_scale | hot_shift
    skew_params: dict = field(default_factory=dict)
    description: str = ""

    def dims(self) -> dict:
        return dict(T=self.T, d_model=self.d_model, d_ff=self.d_ff, E=self.E, K=self.K,
                    capacity_factor=self.capacity_factor)


_CALIB_PATH = os.path.join(os.path.dirname(__file__), "workloads.json")


def _load_calibration() -> dict:
    try:
        with open(_CALIB_PATH) as f:
            return json.load(f)
    except FileNotFoundError:
        return {}


def workloads() -> dict:
    cal = _load_calibration()
    w = {
        "tiny": Workload(
            "tiny", T=64, d_model=128, d_ff=256, E=8, K=2, seed=0,
            description="tiny MoE layer: T=64, d=128, f=256, E=8, top-2, SwiGLU, no bias, no capacity"),
        "mixtral_decode": Workload(
            "mixtral_decode", T=256, d_model=4096, d_ff=14336, E=8, K=2, seed=1,
            description="Mixtral-8x7B-shaped layer, decode-sized batch (T=256), near-uniform routing"),
        "mixtral_prefill": Workload(
            "mixtral_prefill", T=16384, d_model=4096, d_ff=14336, E=8, K=2, seed=2,
            skew="col_scale", skew_params=cal.get("mixtral_prefill", {}),
            description="Mixtral-8x7B-shaped layer, prefill-sized batch (T=16384), ~20% count CV"),
        "qwen_capacity": Workload(
            "qwen_capacity", T=8192, d_model=2048, d_ff=1408, E=60, K=4, capacity_factor=1.0, seed=3,
            skew="hot_shift", skew_params=cal.get("qwen_capacity", {}),
            description="Qwen-MoE-like layer, E=60 top-4, capacity factor 1.0, 6 hot experts (~4x mean)"),
        "deepseek_bias": Workload(
            "deepseek_bias", T=4096, d_model=7168, d_ff=2048, E=256, K=8, seed=4,
            use_bias=True, alpha=1e-3, steps=10,
            skew="col_scale", skew_params=cal.get("deepseek_bias", {}),
            description="DeepSeek-V3-like layer, E=256 top-8, aux-free bias, Zipf(1.1) popularity"),
    }
    return w


def get_workload(name: str) -> Workload:
    return workloads()[name]


def router_col_transform(wl: Workload, device="cpu"):
    """(col_scale, col_shift) applied to the router weight columns."""
    E = wl.E
    if wl.skew == "col_scale" and "scales" in wl.skew_params:
        # a workload reduced to its first E experts (a profiling case) keeps their scales
        return torch.tensor(wl.skew_params["scales"][:E], dtype=torch.float32, device=device), None
    if wl.skew == "hot_shift" and "shift" in wl.skew_params:
        shift = torch.zeros(E, dtype=torch.float32)
        for e in wl.skew_params["hot"]:
            if e < E:
                shift[e] = float(wl.skew_params["shift"])
        return None, shift.to(device)
    return None, None


def make_x(wl: Workload, step: int = 0, device="cpu") -> torch.Tensor:
    seed = wl.seed if step == 0 else wl.seed * 1000 + step
    return normal_bf16((wl.T, wl.d_model), seed, STREAM_X, wl.x_std, device)


def make_router(wl: Workload, device="cpu", col_scale=None, col_shift=None) -> torch.Tensor:
    if col_scale is None and col_shift is None:
        col_scale, col_shift = router_col_transform(wl, device)
    return normal_bf16((wl.d_model, wl.E), wl.seed, STREAM_WR, wl.w_std, device,
                       col_scale=col_scale, col_shift=col_shift)


def make_expert_weights(wl: Workload, device="cpu", experts=None):
    """(W1, W3, W2): W1, W3 [E, d, f], W2 [E, f, d] bf16.

    With ``experts`` (a list of expert ids) only those slabs are returned
    (stacked in that order); each slab is regenerated from its own element
    offsets, so it equals the corresponding slab of the full tensors.
    """
    E, d, f = wl.E, wl.d_model, wl.d_ff
    ids = list(range(E)) if experts is None else [int(e) for e in experts]
    n1 = d * f
    outs = []
    for stream, shape in ((STREAM_W1, (d, f)), (STREAM_W3, (d, f)), (STREAM_W2, (f, d))):
        if experts is None:
            outs.append(normal_bf16((E,) + shape, wl.seed, stream, wl.w_std, device))
        else:
            t = torch.empty((len(ids),) + shape, dtype=torch.bfloat16, device=device)
            for j, e in enumerate(ids):
                t[j] = _normal_slab(shape, wl.seed, stream, wl.w_std, device, e * n1)
            outs.append(t)
    return tuple(outs)


def _normal_slab(shape, seed, stream, std, device, offset):
    numel = 1
    for s in shape:
        numel *= s
    out = torch.empty(numel, dtype=torch.bfloat16, device=device)
    std32 = torch.tensor(std, dtype=torch.float32, device=device)
    pos, chunk = 0, 1 << 24
    while pos < numel:
        take = min(chunk, numel - pos)
        out[pos:pos + take] = (normal_f32(take, seed, stream, device, offset + pos) * std32).to(torch.bfloat16)
        pos += take
    return out.view(shape)


def bf16_to_f64(t: torch.Tensor):
    """bf16 tensor -> numpy float64 array (exact)."""
    return t.detach().to("cpu", torch.float32).double().numpy()
