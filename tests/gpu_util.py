"""Helpers shared by the GPU parity tests (inputs, oracle calls, tolerances).

Inputs come from ``moe_layer_gemm_b200.synth``; expected values come from
``oracle.moe_oracle`` run on copies of the same inputs.  Nothing computed by
the CUDA library is ever fed to the oracle: where fp32 and fp64 logits may
rank two experts differently (a near tie), the test compares what is unique
and checks that the library's choice is a valid one.
"""
from __future__ import annotations

import numpy as np
import torch

from moe_layer_gemm_b200 import abi, synth
from oracle import moe_oracle as O

# Layer output tolerance against the fp64 oracle (bf16 storage, fp32 accumulation).
Y_MAX_ABS = 2e-2
Y_REL_L2 = 5e-3
# Against the oracle that also rounds H to bf16 (same rounding point as the
# kernels): only elements of H whose fp32 and fp64 values straddle a bf16
# rounding boundary differ (by one bf16 ulp), so the bar is tighter than the
# main one but must allow a few such flips per row.
Y_MIRROR_MAX_ABS = 1e-2
Y_MIRROR_REL_L2 = 5e-4
W_TOL = 2e-6      # renormalised weights (fp32 expf vs fp64 exp)
P_TOL = 2e-6      # mean router probabilities


def dev():
    return torch.device("cuda", 0)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close_y(y_gpu: np.ndarray, y_ref: np.ndarray, max_abs=Y_MAX_ABS, rl2=Y_REL_L2, what="y"):
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite values"
    err = np.abs(y_gpu - y_ref)
    ma, r = float(err.max()) if err.size else 0.0, rel_l2(y_gpu, y_ref)
    assert ma <= max_abs and r <= rl2, f"{what}: max-abs {ma:.3e} (tol {max_abs}), rel-L2 {r:.3e} (tol {rl2})"
    return ma, r


def ambiguous_tokens(l64: np.ndarray, bound: np.ndarray, K: int, bias32=None) -> np.ndarray:
    """Tokens whose top-K set or order could differ under logit errors <= bound.

    A token is unambiguous when every adjacent pair in its sorted (biased)
    logits, down to position K, is separated by more than the two values'
    bounds plus one fp32 ulp of rounding at each end.
    """
    l = l64 + (0 if bias32 is None else np.asarray(bias32, np.float64)[None, :])
    T, E = l.shape
    order = np.argsort(-l, axis=1, kind="stable")
    ls = np.take_along_axis(l, order, 1)
    bs = np.take_along_axis(bound, order, 1)
    ulp = np.abs(ls) * 2.0 ** -23 + 1e-30
    upto = min(K + 1, E)
    amb = np.zeros(T, dtype=bool)
    for j in range(upto - 1):
        gap = ls[:, j] - ls[:, j + 1]
        amb |= gap <= (bs[:, j] + bs[:, j + 1] + 2 * ulp[:, j] + 2 * ulp[:, j + 1])
    return amb


def check_routing_validity(idx_gpu: np.ndarray, l64: np.ndarray, bound: np.ndarray, K: int, bias32=None):
    """The library's selection is a valid top-K for some logits within the bound."""
    l = l64 + (0 if bias32 is None else np.asarray(bias32, np.float64)[None, :])
    T, E = l.shape
    slack = bound + np.abs(l) * 2.0 ** -22 + 1e-30
    for t in range(T):
        sel = idx_gpu[t].tolist()
        assert len(set(sel)) == K and all(0 <= e < E for e in sel)
        rest = [e for e in range(E) if e not in sel]
        if rest:
            lo = min(l[t, e] + slack[t, e] for e in sel)
            hi = max(l[t, e] - slack[t, e] for e in rest)
            assert lo >= hi, f"token {t}: selected {sel} cannot beat the best unselected expert"


def uncertain_tokens(idx_a: np.ndarray, idx_b: np.ndarray, E: int, capacity) -> np.ndarray:
    """Tokens whose outputs may legitimately differ between two routings.

    Tokens whose selected sets differ, plus (with a capacity) every token
    routed to an expert after the first token where that expert's
    membership differs, since its rank and drop decision can shift.
    """
    T, K = idx_a.shape
    sa = [set(r) for r in idx_a.tolist()]
    sb = [set(r) for r in idx_b.tolist()]
    unc = np.array([sa[t] != sb[t] for t in range(T)])
    if capacity is None or not unc.any():
        return unc
    first = np.full(E, T)
    for t in np.nonzero(unc)[0]:
        for e in sa[t] ^ sb[t]:
            first[e] = min(first[e], t)
    for t in range(T):
        if any(t >= first[e] for e in sa[t] | sb[t]):
            unc[t] = True
    return unc


class LayerInputs:
    """One workload's inputs on the GPU plus host copies for the oracle."""

    def __init__(self, wl: synth.Workload, step: int = 0, T: int | None = None, pack: bool = True):
        d = dev()
        self.wl = wl
        self.T = wl.T if T is None else T
        self.dims = abi.Dims(self.T, wl.d_model, wl.d_ff, wl.E, wl.K, wl.capacity_factor)
        x = synth.make_x(wl, step, device=d)
        self.x = x[: self.T].contiguous()
        self.Wr = synth.make_router(wl, device=d)
        self.W1, self.W3, self.W2 = synth.make_expert_weights(wl, device=d)
        if pack:
            self.W13p, self.W2p = abi.pack_weights(self.dims, self.W1, self.W3, self.W2)
            torch.cuda.synchronize()
        self.ws = abi.alloc_workspace(self.dims)

    def host(self):
        return f64(self.x), f64(self.Wr)

    def expert_slabs(self, experts):
        """fp64 host copies of the listed experts' weights (inputs, not results)."""
        ids = torch.tensor(list(experts), dtype=torch.long, device=self.W1.device)
        return f64(self.W1[ids]), f64(self.W3[ids]), f64(self.W2[ids])


def oracle_layer(inp: LayerInputs, bias32=None, tokens=None, h_round=None, alpha=0.0):
    """The oracle on the same inputs; with ``tokens`` only those rows of y."""
    x64, Wr64 = inp.host()
    E = inp.wl.E
    if tokens is None:
        W1, W3, W2 = inp.expert_slabs(range(E))
        return O.moe_layer(x64, Wr64, W1, W3, W2, inp.wl.K, inp.wl.capacity_factor, bias32=bias32,
                           alpha=alpha, h_round=h_round)
    # routing for all tokens, FFN only for the sampled ones: fetch only the
    # experts those tokens use (the oracle's own routing decides which)
    l32 = O.router_logits(x64, Wr64).astype(np.float32)
    idx, _, _ = O.route_from_logits_f32(l32, inp.wl.K, bias32)
    used = sorted({int(e) for t in tokens for e in idx[t]})

    class Lazy:
        """Expert slabs fetched (as inputs) and widened to fp64 one at a time."""

        def __init__(self, src):
            self.src = src
            self.shape = tuple(src.shape)

        def __getitem__(self, e):
            assert int(e) in used
            return f64(self.src[int(e)])

    return O.moe_layer(x64, Wr64, Lazy(inp.W1), Lazy(inp.W3), Lazy(inp.W2), inp.wl.K,
                       inp.wl.capacity_factor, bias32=bias32, alpha=alpha, tokens=tokens, h_round=h_round)


def oracle_routing(inp: LayerInputs, bias32=None):
    """The oracle's own routing of the whole batch (fp32 decisions on its
    correctly rounded logits) plus the rigorous logit error bound; computed
    from the inputs only."""
    x64, Wr64 = inp.host()
    K, E = inp.wl.K, inp.wl.E
    l64 = O.router_logits(x64, Wr64)
    idx, _, _ = O.route_from_logits_f32(l64.astype(np.float32), K, bias32)
    C = O.capacity(inp.T, K, E, inp.wl.capacity_factor)
    disp = O.dispatch(idx, E, C)
    bound = 2.0 * O.dot_error_bound(x64, Wr64) + np.abs(l64) * 2.0 ** -23
    return idx, disp, l64, bound


def covering_sample(inp: LayerInputs, S: int, bias32=None, seed: int = 0, per_expert: int = 2):
    """Sorted token ids, at least min(S, T) of them: for every expert with
    kept rows under the oracle's routing, the `per_expert` earliest tokens
    that keep a slot on it, unambiguous ones (top-K fixed under the logit
    error bound) first, so that one token routed differently by the library
    does not lose the expert (early tokens also keep their capacity ranks
    when a later routing differs); the rest seeded uniform draws.  Also
    returns the set of experts with kept rows."""
    idx, disp, l64, bound = oracle_routing(inp, bias32)
    T, K, E = inp.T, inp.wl.K, inp.wl.E
    amb = ambiguous_tokens(l64, bound, K, bias32)
    inv = disp["inv"]
    need = {e for e in range(E) if disp["kept"][e] > 0}
    cand = {e: [] for e in need}
    for t in range(T):
        for k in range(K):
            if inv[t, k] >= 0:
                cand[int(idx[t, k])].append(t)
    chosen = set()
    for e in need:
        ts = sorted(cand[e], key=lambda t: (bool(amb[t]), t))
        chosen.update(ts[:per_expert])
    rng = np.random.default_rng(seed)
    rest = [t for t in rng.permutation(T).tolist() if t not in chosen]
    chosen.update(rest[: max(0, S - len(chosen))])
    return sorted(chosen), need


def experts_compared(rows, idx_ref: np.ndarray, inv_ref: np.ndarray) -> set:
    """Experts that hold a kept slot of at least one compared token."""
    return {int(idx_ref[t, k]) for t in rows for k in range(idx_ref.shape[1]) if inv_ref[t, k] >= 0}

