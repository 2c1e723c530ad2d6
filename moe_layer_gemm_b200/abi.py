"""ctypes binding of the C ABI in include/moe_b200.h.

Argument marshalling only: every function takes torch tensors (device
memory owned by the caller) or None, checks dtype / device / contiguity,
passes raw pointers and the current CUDA stream to the library and raises
``MoEError`` on a non-zero status.  All computation happens in the CUDA
kernels of ``lib/libmoe_b200.so``; there is no fallback of any kind, so a
missing or unloadable library is an error.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libmoe_b200.so")

MOE_OK = 0
MOE_EINVAL = -1
MOE_EUNSUPPORTED = -2
MOE_ECUDA = -3
MOE_EWORKSPACE = -4
MOE_ETIMEOUT = -5
MOE_ESCRATCH = -6
MOE_EINDEX = -7
MOE_SLOT_SKIP = -2  # slot table entry that leaves an expert out of moe_expert_ffn_slots

EXPORTED = [
    "moe_status_str", "moe_version", "moe_capacity", "moe_workspace_size", "moe_reset_device_status",
    "moe_get_device_status", "moe_pack_weights", "moe_route", "moe_route_from_logits", "moe_permute",
    "moe_expert_ffn", "moe_combine", "moe_load_stats", "moe_bias_update", "moe_layer_forward",
    "moe_layer_launch_count", "moe_packed_weight_bytes", "moe_permute_noalloc", "moe_ffn_kernel",
    "moe_chunked_workspace_size", "moe_layer_forward_chunked", "moe_layer_chunked_launch_count",
    "moe_test_set_wait_limits", "moe_ep_regroup", "moe_int4_bytes", "moe_int4_pack", "moe_int4_unpack",
    "moe_expert_ffn_slots",
]
NUM_STAGE_EVENTS = 6


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


class moe_dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("K", ctypes.c_int32), ("capacity_factor", ctypes.c_double)]


class moe_layer_outputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("topk_idx", "topk_w", "logits", "counts", "kept", "offsets", "inv", "n_dropped", "f", "P", "aux",
                 "stage_events", "P_topk", "aux_topk", "z_loss")]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run python -m moe_layer_gemm_b200.build)")
    lib = ctypes.CDLL(path)
    P, I, I64, SZ, F, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_double
    dims_p = ctypes.POINTER(moe_dims)
    sig = {
        "moe_status_str": (ctypes.c_char_p, [I]),
        "moe_version": (I, []),
        "moe_capacity": (I64, [dims_p]),
        "moe_workspace_size": (I, [dims_p, ctypes.POINTER(SZ)]),
        "moe_reset_device_status": (I, [P, P]),
        "moe_get_device_status": (I, [P, P, ctypes.POINTER(I), ctypes.POINTER(I)]),
        "moe_pack_weights": (I, [dims_p, P, P, P, P, P, P]),
        "moe_route": (I, [dims_p, P, P, P, P, P, P, P, P, SZ, P]),
        "moe_route_from_logits": (I, [dims_p, P, P, P, P, P, P, SZ, P]),
        "moe_permute": (I, [dims_p, P, P, P, P, P, P, P, P, P, P, SZ, P]),
        "moe_expert_ffn": (I, [dims_p, P, P, P, P, P, P, P, SZ, P]),
        "moe_combine": (I, [dims_p, P, P, P, P, I, P]),
        "moe_load_stats": (I, [dims_p, P, P, P, P, P]),
        "moe_bias_update": (I, [dims_p, P, F, P, P]),
        "moe_layer_forward": (I, [dims_p, P, P, P, F, P, P, P, I, ctypes.POINTER(moe_layer_outputs), P, SZ, P]),
        "moe_layer_launch_count": (I, [dims_p, I, I]),
        "moe_packed_weight_bytes": (I, [dims_p, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]),
        "moe_permute_noalloc": (I, [dims_p, P, P, P, P, P, P, P, P, P, P]),
        "moe_ffn_kernel": (I, [dims_p]),
        "moe_chunked_workspace_size": (I, [dims_p, ctypes.c_int64, ctypes.POINTER(SZ)]),
        "moe_layer_chunked_launch_count": (I, [dims_p, ctypes.c_int64, I, I]),
        "moe_layer_forward_chunked": (I, [dims_p, ctypes.c_int64, P, P, P, F, P, P, P, I,
                                          ctypes.POINTER(moe_layer_outputs), P, SZ, P]),
        "moe_test_set_wait_limits": (I, [ctypes.c_int64, ctypes.c_int64, I]),
        "moe_ep_regroup": (I, [I, I, P, I64, I, P, P, P, P, P]),
        "moe_int4_bytes": (I, [dims_p, ctypes.POINTER(SZ), ctypes.POINTER(SZ), ctypes.POINTER(SZ),
                               ctypes.POINTER(SZ)]),
        "moe_int4_pack": (I, [dims_p, P, P, P, P, P, P, P, P]),
        "moe_int4_unpack": (I, [dims_p, I, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                P, P, P, P, I, P, P, P]),
        "moe_expert_ffn_slots": (I, [dims_p, P, P, P, I, P, P, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


@dataclass
class Dims:
    T: int
    d_model: int
    d_ff: int
    E: int
    K: int
    capacity_factor: float = 0.0

    def c(self) -> moe_dims:
        return moe_dims(self.T, self.d_model, self.d_ff, self.E, self.K, float(self.capacity_factor))


def _dims(d) -> moe_dims:
    if isinstance(d, moe_dims):
        return d
    if isinstance(d, Dims):
        return d.c()
    if isinstance(d, dict):
        return Dims(**d).c()
    return Dims(d.T, d.d_model, d.d_ff, d.E, d.K, getattr(d, "capacity_factor", 0.0)).c()


def _ptr(t: Optional[torch.Tensor], dtype=None, name: str = "") -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != MOE_OK:
        msg = load().moe_status_str(status).decode()
        raise MoEError(fn, status, msg)


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32


def moe_status_str(status: int) -> str:
    return load().moe_status_str(status).decode()


def moe_version() -> int:
    return load().moe_version()


def moe_test_set_wait_limits(wait_polls: int = 0, dependency_polls: int = 0, dependency_never_ready: bool = False):
    """Test-only: poll limits of the expert GEMMs' bounded waits (0 = default)
    and an unreachable down-projection readiness target (see the header)."""
    _check("moe_test_set_wait_limits", load().moe_test_set_wait_limits(
        ctypes.c_int64(wait_polls), ctypes.c_int64(dependency_polls), int(bool(dependency_never_ready))))


def moe_capacity(dims) -> int:
    return int(load().moe_capacity(ctypes.byref(_dims(dims))))


def moe_workspace_size(dims) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size", load().moe_workspace_size(ctypes.byref(_dims(dims)), ctypes.byref(n)))
    return int(n.value)


def moe_chunked_workspace_size(dims, chunk_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_chunked_workspace_size", load().moe_chunked_workspace_size(
        ctypes.byref(_dims(dims)), ctypes.c_int64(chunk_tokens), ctypes.byref(n)))
    return int(n.value)


def alloc_chunked_workspace(dims, chunk_tokens: int, device="cuda") -> torch.Tensor:
    """Caller-owned workspace for moe_layer_forward_chunked."""
    return torch.zeros(moe_chunked_workspace_size(dims, chunk_tokens), dtype=torch.uint8, device=device)


def alloc_workspace(dims, device="cuda") -> torch.Tensor:
    """Caller-owned workspace (uint8) of moe_workspace_size(dims) bytes."""
    return torch.zeros(moe_workspace_size(dims), dtype=torch.uint8, device=device)


def moe_reset_device_status(ws: torch.Tensor, stream=None):
    _check("moe_reset_device_status", load().moe_reset_device_status(_ptr(ws, None, "ws"), _stream(stream)))


def moe_get_device_status(ws: torch.Tensor, stream=None):
    s, d = ctypes.c_int(0), ctypes.c_int(0)
    _check("moe_get_device_status", load().moe_get_device_status(_ptr(ws, None, "ws"), _stream(stream),
                                                                 ctypes.byref(s), ctypes.byref(d)))
    return s.value, d.value


def moe_pack_weights(dims, W1, W3, W2, W13p, W2p, stream=None):
    _check("moe_pack_weights", load().moe_pack_weights(
        ctypes.byref(_dims(dims)), _ptr(W1, BF16, "W1"), _ptr(W3, BF16, "W3"), _ptr(W2, BF16, "W2"),
        _ptr(W13p, BF16, "W13p"), _ptr(W2p, BF16, "W2p"), _stream(stream)))


def moe_route(dims, x, Wr, bias, logits, topk_idx, topk_w, prob_mean, ws, stream=None):
    _check("moe_route", load().moe_route(
        ctypes.byref(_dims(dims)), _ptr(x, BF16, "x"), _ptr(Wr, BF16, "Wr"), _ptr(bias, F32, "bias"),
        _ptr(logits, F32, "logits"), _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"),
        _ptr(prob_mean, F32, "prob_mean"), _ptr(ws, None, "ws"), ws.numel(), _stream(stream)))


def moe_route_from_logits(dims, logits, bias, topk_idx, topk_w, prob_mean, ws, stream=None):
    _check("moe_route_from_logits", load().moe_route_from_logits(
        ctypes.byref(_dims(dims)), _ptr(logits, F32, "logits"), _ptr(bias, F32, "bias"),
        _ptr(topk_idx, I32, "topk_idx"), _ptr(topk_w, F32, "topk_w"), _ptr(prob_mean, F32, "prob_mean"),
        _ptr(ws, None, "ws"), ws.numel(), _stream(stream)))


def moe_permute(dims, topk_idx, x, counts, kept, offsets, inv, src, x_perm, n_dropped, ws, stream=None):
    _check("moe_permute", load().moe_permute(
        ctypes.byref(_dims(dims)), _ptr(topk_idx, I32, "topk_idx"), _ptr(x, BF16, "x"),
        _ptr(counts, I32, "counts"), _ptr(kept, I32, "kept"), _ptr(offsets, I32, "offsets"),
        _ptr(inv, I32, "inv"), _ptr(src, I32, "src"), _ptr(x_perm, BF16, "x_perm"),
        _ptr(n_dropped, I32, "n_dropped"), _ptr(ws, None, "ws"), ws.numel(), _stream(stream)))


def moe_permute_noalloc(dims, topk_idx, x, counts, kept, offsets, inv, src, x_perm, n_dropped, stream=None):
    """moe_permute without a workspace (scratch held inside the library)."""
    _check("moe_permute_noalloc", load().moe_permute_noalloc(
        ctypes.byref(_dims(dims)), _ptr(topk_idx, I32, "topk_idx"), _ptr(x, BF16, "x"),
        _ptr(counts, I32, "counts"), _ptr(kept, I32, "kept"), _ptr(offsets, I32, "offsets"),
        _ptr(inv, I32, "inv"), _ptr(src, I32, "src"), _ptr(x_perm, BF16, "x_perm"),
        _ptr(n_dropped, I32, "n_dropped"), _stream(stream)))


def moe_expert_ffn(dims, x_perm, offsets, W13p, W2p, h, y_perm, ws, stream=None):
    _check("moe_expert_ffn", load().moe_expert_ffn(
        ctypes.byref(_dims(dims)), _ptr(x_perm, BF16, "x_perm"), _ptr(offsets, I32, "offsets"),
        _ptr(W13p, BF16, "W13p"), _ptr(W2p, BF16, "W2p"), _ptr(h, BF16, "h"), _ptr(y_perm, F32, "y_perm"),
        _ptr(ws, None, "ws"), ws.numel(), _stream(stream)))


def _y_arg(y):
    """Pointer and y_is_bf16 flag of a layer output (fp32 or bf16 tensor)."""
    if y is not None and y.dtype == BF16:
        return _ptr(y, BF16, "y"), 1
    return _ptr(y, F32, "y"), 0


def moe_combine(dims, y_perm, inv, topk_w, y, stream=None):
    """y may be fp32 or bf16 (the fp32 sum rounded to nearest even)."""
    yp, yb = _y_arg(y)
    _check("moe_combine", load().moe_combine(
        ctypes.byref(_dims(dims)), _ptr(y_perm, F32, "y_perm"), _ptr(inv, I32, "inv"),
        _ptr(topk_w, F32, "topk_w"), yp, yb, _stream(stream)))


def moe_load_stats(dims, counts, prob_mean, f, aux, stream=None):
    _check("moe_load_stats", load().moe_load_stats(
        ctypes.byref(_dims(dims)), _ptr(counts, I32, "counts"), _ptr(prob_mean, F32, "prob_mean"),
        _ptr(f, F32, "f"), _ptr(aux, F32, "aux"), _stream(stream)))


def moe_bias_update(dims, counts, alpha: float, bias, stream=None):
    _check("moe_bias_update", load().moe_bias_update(
        ctypes.byref(_dims(dims)), _ptr(counts, I32, "counts"), ctypes.c_float(alpha), _ptr(bias, F32, "bias"),
        _stream(stream)))


def moe_layer_forward(dims, x, Wr, bias, alpha: float, W13p, W2p, y, ws, outputs: Optional[dict] = None,
                      stream=None, stage_events=None):
    """The whole layer.  ``y`` is fp32 or bf16; ``outputs`` maps
    moe_layer_outputs field names to tensors; ``stage_events`` is a sequence
    of NUM_STAGE_EVENTS recorded torch.cuda.Event objects (or None)."""
    o = None
    keep = None
    if outputs or stage_events is not None:
        o = moe_layer_outputs()
        for k, t in (outputs or {}).items():
            setattr(o, k, _ptr(t, None, k))
        if stage_events is not None:
            if len(stage_events) != NUM_STAGE_EVENTS:
                raise ValueError("stage_events needs NUM_STAGE_EVENTS events")
            keep = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*[ev.cuda_event for ev in stage_events])
            o.stage_events = ctypes.cast(keep, ctypes.c_void_p)
    _check("moe_layer_forward", load().moe_layer_forward(
        ctypes.byref(_dims(dims)), _ptr(x, BF16, "x"), _ptr(Wr, BF16, "Wr"), _ptr(bias, F32, "bias"),
        ctypes.c_float(alpha), _ptr(W13p, BF16, "W13p"), _ptr(W2p, BF16, "W2p"), *_y_arg(y),
        ctypes.byref(o) if o is not None else None, _ptr(ws, None, "ws"), ws.numel(), _stream(stream)))


def moe_layer_forward_chunked(dims, chunk_tokens: int, x, Wr, bias, alpha: float, W13p, W2p, y, ws,
                              outputs: Optional[dict] = None, stream=None):
    """The layer in chunks of at most ``chunk_tokens`` tokens (see the header)."""
    o = None
    if outputs:
        o = moe_layer_outputs()
        for k, t in outputs.items():
            setattr(o, k, _ptr(t, None, k))
    _check("moe_layer_forward_chunked", load().moe_layer_forward_chunked(
        ctypes.byref(_dims(dims)), ctypes.c_int64(chunk_tokens), _ptr(x, BF16, "x"), _ptr(Wr, BF16, "Wr"),
        _ptr(bias, F32, "bias"), ctypes.c_float(alpha), _ptr(W13p, BF16, "W13p"), _ptr(W2p, BF16, "W2p"),
        *_y_arg(y), ctypes.byref(o) if o is not None else None, _ptr(ws, None, "ws"), ws.numel(),
        _stream(stream)))


def moe_layer_chunked_launch_count(dims, chunk_tokens: int, stats: bool, bias_update: bool) -> int:
    n = load().moe_layer_chunked_launch_count(ctypes.byref(_dims(dims)), ctypes.c_int64(chunk_tokens), int(stats),
                                              int(bias_update))
    if n < 0:
        raise MoEError("moe_layer_chunked_launch_count", n, "invalid arguments")
    return n


def moe_layer_launch_count(dims, stats: bool, bias_update: bool) -> int:
    n = load().moe_layer_launch_count(ctypes.byref(_dims(dims)), int(stats), int(bias_update))
    if n < 0:
        raise MoEError("moe_layer_launch_count", n, "invalid dims")
    return n


FFN_KERNELS = ("grouped_gemm_kernel", "grouped_gemm_2sm_kernel")


def moe_ffn_kernel(dims) -> str:
    """Name of the grouped-GEMM kernel the expert FFN launches for these dims."""
    k = load().moe_ffn_kernel(ctypes.byref(_dims(dims)))
    if k < 0:
        raise MoEError("moe_ffn_kernel", k, "invalid dims")
    return FFN_KERNELS[k]


def moe_ep_regroup(n_ranks: int, E_local: int, recv_counts, rows_in, rows_out, offsets, row_of, stream=None):
    """Regroup the rows a rank received (source-major) by local expert (see the header)."""
    n = 0 if rows_in is None else int(rows_in.shape[0])
    d = int(rows_out.shape[1]) if rows_out is not None and rows_out.dim() == 2 else 8
    _check("moe_ep_regroup", load().moe_ep_regroup(
        int(n_ranks), int(E_local), _ptr(recv_counts, I32, "recv_counts"), ctypes.c_int64(n), d,
        _ptr(rows_in, BF16, "rows_in") if n else None, _ptr(rows_out, BF16, "rows_out") if n else None,
        _ptr(offsets, I32, "offsets"), _ptr(row_of, I32, "row_of") if n else None, _stream(stream)))


def moe_int4_bytes(dims):
    """(q13, s13, q2, s2) byte counts of all experts' INT4 codes and scales."""
    v = [ctypes.c_size_t(0) for _ in range(4)]
    _check("moe_int4_bytes", load().moe_int4_bytes(ctypes.byref(_dims(dims)), *[ctypes.byref(x) for x in v]))
    return tuple(int(x.value) for x in v)


def _any_ptr(t, dtype, name):
    """Pointer of a device tensor or of a page-locked host tensor."""
    if t.device.type == "cpu":
        if not t.is_pinned():
            raise ValueError(f"{name}: a host tensor must be page-locked (pin_memory)")
        if t.dtype != dtype or not t.is_contiguous():
            raise TypeError(f"{name}: expected a contiguous {dtype} tensor")
        return t.data_ptr()
    return _ptr(t, dtype, name)


def moe_int4_pack(dims, W1, W3, W2, q13, s13, q2, s2, stream=None):
    _check("moe_int4_pack", load().moe_int4_pack(
        ctypes.byref(_dims(dims)), _ptr(W1, BF16, "W1"), _ptr(W3, BF16, "W3"), _ptr(W2, BF16, "W2"),
        _ptr(q13, torch.uint8, "q13"), _ptr(s13, F32, "s13"), _ptr(q2, torch.uint8, "q2"), _ptr(s2, F32, "s2"),
        _stream(stream)))


def moe_int4_unpack(dims, experts, slots, q13, s13, q2, s2, n_slots: int, W13c, W2c, stream=None):
    """Expand experts[j]'s INT4 codes into cache slot slots[j] (host lists)."""
    n = len(experts)
    if n != len(slots):
        raise ValueError("experts and slots differ in length")
    if n == 0:
        return
    je = (ctypes.c_int32 * n)(*[int(e) for e in experts])
    js = (ctypes.c_int32 * n)(*[int(s) for s in slots])
    _check("moe_int4_unpack", load().moe_int4_unpack(
        ctypes.byref(_dims(dims)), n, je, js, _any_ptr(q13, torch.uint8, "q13"), _any_ptr(s13, F32, "s13"),
        _any_ptr(q2, torch.uint8, "q2"), _any_ptr(s2, F32, "s2"), int(n_slots), _ptr(W13c, BF16, "W13c"),
        _ptr(W2c, BF16, "W2c"), _stream(stream)))


def moe_expert_ffn_slots(dims, x_perm, offsets, expert_slot, n_slots: int, W13c, W2c, h, y_perm, ws, stream=None):
    _check("moe_expert_ffn_slots", load().moe_expert_ffn_slots(
        ctypes.byref(_dims(dims)), _ptr(x_perm, BF16, "x_perm"), _ptr(offsets, I32, "offsets"),
        _ptr(expert_slot, I32, "expert_slot"), int(n_slots), _ptr(W13c, BF16, "W13c"), _ptr(W2c, BF16, "W2c"),
        _ptr(h, BF16, "h"), _ptr(y_perm, F32, "y_perm"), _ptr(ws, None, "ws"), ws.numel(), _stream(stream)))


# ---------------------------------------------------------------- helpers

def moe_packed_weight_bytes(dims):
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check("moe_packed_weight_bytes",
           load().moe_packed_weight_bytes(ctypes.byref(_dims(dims)), ctypes.byref(a), ctypes.byref(b)))
    return int(a.value), int(b.value)


def pack_weights(dims, W1, W3, W2, stream=None):
    """Allocate and fill the packed expert weights (W13p, W2p): flat bf16
    buffers in the library's tiled layout."""
    n13, n2 = moe_packed_weight_bytes(dims)
    W13p = torch.empty(n13 // 2, dtype=BF16, device=W1.device)
    W2p = torch.empty(n2 // 2, dtype=BF16, device=W1.device)
    moe_pack_weights(dims, W1, W3, W2, W13p, W2p, stream)
    return W13p, W2p
