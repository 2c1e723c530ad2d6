"""CPU oracle for one Mixture-of-Experts FFN layer forward pass.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import or run this module.  The product path
(the CUDA library and its binding) never calls it, and it shares no code with
that path: it imports numpy and the Python standard library only.

Plain, slow and meant to be checked by eye against the pages:
  [P2] "MoE computation notes", cf-1.com/news/5905749
  [P3] "MoE inference engineering in practice", ybb.press/quantum-computing/18594
  [P1] "MoE serving essay", dpshk.com/news/3211971

Floating point is fp64 on the bf16-rounded inputs, except where fp32 decides
an integer (top-K selection on fp32 logits) or where the method is itself an
fp32 recurrence (the aux-free bias update); there the oracle works in fp32 as
the kernels do.  Readings of passages that are silent or ambiguous are marked
READING and listed in the design notes.

Every function is pinned by the oracle's own tests against closed forms,
invariants and brute force (tests/test_oracle_pins.py); none is "parity
unpinned".
"""
from __future__ import annotations

from fractions import Fraction
import math

import numpy as np


# ---------------------------------------------------------------------------
# a1. Router logits
# ---------------------------------------------------------------------------

def router_logits(x: np.ndarray, Wr: np.ndarray, bias=None) -> np.ndarray:
    """logits[t, e] = sum_d x[t, d] * Wr[d, e]  (+ bias[e]), in fp64.

    [P2] section 1.2 (router_forward: a linear map x @ router_weight with
    router_weight laid out [hidden_size, num_experts]); [P3] section 1.2
    (the aux-free variant routes on gate(x) + bias).
    """
    x = np.asarray(x, dtype=np.float64)
    Wr = np.asarray(Wr, dtype=np.float64)
    out = x @ Wr
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)[None, :]
    return out


def softmax_rows(logits: np.ndarray) -> np.ndarray:
    """Full softmax over all E experts per token, fp64.

    [P2] section 1.1 / section 2 step 1: s = softmax(x W_r).
    """
    l = np.asarray(logits, dtype=np.float64)
    m = l.max(axis=1, keepdims=True)
    p = np.exp(l - m)
    return p / p.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# a2. Top-K selection and renormalisation
# ---------------------------------------------------------------------------

def topk_select(logits: np.ndarray, K: int) -> np.ndarray:
    """[T, K] int32: the K largest logits per token, in descending order.

    [P2] section 2 step 2 and [P3] section 1 (torch.topk on the logits).
    READING (tie rule, silent on the pages): equal values rank the lower
    expert index first; -0.0 and +0.0 are equal.  Values are compared in the
    dtype given (fp32 logits are compared as fp32).
    """
    l = np.asarray(logits)
    T, E = l.shape
    if not (1 <= K <= E):
        raise ValueError("need 1 <= K <= E")
    if not np.all(np.isfinite(l)):
        raise ValueError("logits must be finite")
    # A stable sort of -value keeps the lower index first among equal values.
    order = np.argsort(-l, axis=1, kind="stable")
    return order[:, :K].astype(np.int32)


def renormalized_weights(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """[T, K] fp64: w_j = exp(l_j - l_max) / sum over the selected of exp(l - l_max).

    [P2] section 2 step 3 and section 2.1 (a second softmax over the K
    selected scores); [P3] section 1 (softmax over the top-K logits).
    READING: the softmax is taken over the K selected *logits*; this equals
    the full-softmax probabilities renormalised over the selected experts.
    """
    l = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(l, idx.astype(np.int64), axis=1)
    m = sel.max(axis=1, keepdims=True)
    e = np.exp(sel - m)
    return e / e.sum(axis=1, keepdims=True)


def route_from_logits_f32(logits32: np.ndarray, K: int, bias32=None):
    """Selection and weights from fp32 logits, deciding in fp32.

    The biased logit is the fp32 sum fl32(l + b) ([P3] section 1.2: route on
    gate(x) + bias); both the selection and the weights use it (READING).
    Returns (idx int32 [T,K], w fp64 [T,K], biased fp32 logits).
    """
    l = np.asarray(logits32, dtype=np.float32)
    if bias32 is not None:
        l = (l + np.asarray(bias32, dtype=np.float32)[None, :]).astype(np.float32)
    idx = topk_select(l, K)
    w = renormalized_weights(l.astype(np.float64), idx)
    return idx, w, l


# ---------------------------------------------------------------------------
# a3. Load statistics
# ---------------------------------------------------------------------------

def expert_counts(idx: np.ndarray, E: int) -> np.ndarray:
    """cnt[e] = number of (token, slot) pairs that selected expert e (pre-drop).

    [P3] section 1.2 (count_tokens_per_expert(selected)).
    """
    cnt = np.zeros(E, dtype=np.int64)
    for e in np.asarray(idx).reshape(-1):
        cnt[int(e)] += 1
    return cnt


def load_stats(counts: np.ndarray, probs: np.ndarray, T: int, K: int):
    """(f, P, aux) with f_i = cnt_i / (T K), P_i = mean_t p_{t,i}, aux = N sum f_i P_i.

    [P2] section 1.2 (aux_loss = N * sum_i f_i * P_i; f_i the selected
    fraction, P_i the router's mean probability) and section 3.2.
    READING: f_i is the share of the T*K selections, so sum f_i = 1; P_i uses
    the unbiased router softmax.  With either f or P uniform, aux = 1.
    """
    E = counts.shape[0]
    f = np.asarray(counts, dtype=np.float64) / float(T * K)
    P = np.asarray(probs, dtype=np.float64).sum(axis=0) / float(T)
    aux = float(E) * float(np.sum(f * P))
    return f, P, aux


def router_z_loss(logits: np.ndarray) -> float:
    """z_loss = (1/T) sum_t (log sum_j exp(s_tj))^2, in fp64.

    [P2] section 3.2 (router z-loss: it keeps the router logits small by
    penalising the square of their log-sum-exp, averaged over the tokens).
    READING: s are the unbiased router logits x W_r, the same ones P_i uses;
    the aux-free bias is a routing adjustment, not router output.
    """
    s = np.asarray(logits, dtype=np.float64)
    m = s.max(axis=1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return float(np.mean(lse * lse))


def topk_load_stats(counts: np.ndarray, idx: np.ndarray, w: np.ndarray, T: int, K: int):
    """(P_topk, aux_topk): the cheaper form of the balance loss that counts
    only the probabilities of the selected experts.

    [P2] section 3.2 (an approximate aux loss that sums only the top-K
    selected probabilities instead of the soft assignment over all experts).
    READING: P~_i = (1/T) * sum over (t, k) with idx[t, k] = i of w[t, k],
    the renormalised top-K weights the router emits; aux_topk =
    N * sum_i f_i P~_i with f_i as in load_stats.
    """
    E = counts.shape[0]
    f = np.asarray(counts, dtype=np.float64) / float(T * K)
    Pt = np.zeros(E)
    for t in range(idx.shape[0]):
        for k in range(idx.shape[1]):
            Pt[int(idx[t, k])] += float(w[t, k])
    Pt /= float(T)
    return Pt, float(E) * float(np.sum(f * Pt))


# ---------------------------------------------------------------------------
# a4. Dispatch with capacity
# ---------------------------------------------------------------------------

def capacity(T: int, K: int, E: int, capacity_factor: float):
    """C = ceil(CF * T * K / E) computed exactly; None when CF <= 0 (no limit).

    [P2] section 3.1 (average load T*K/E; capacity = a multiple of it).
    READING: ceiling of the exact rational value of the given double.
    """
    if capacity_factor is None or capacity_factor <= 0:
        return None
    q = Fraction(capacity_factor) * T * K / E
    return int(math.ceil(q))


def dispatch(idx: np.ndarray, E: int, C=None):
    """Group assignments by expert, in token order, and apply the capacity.

    [P2] section 2.1 (dispatch: permute tokens so each expert's tokens are
    adjacent, by sort and cumsum) and section 3.1 (assignments beyond an
    expert's capacity are dropped).
    READING: the rank of (t, k) on expert e is the number of earlier tokens
    t' < t that also chose e; it is kept iff rank < C.  Rows of x_perm are
    expert-major, token-ascending.

    Returns dict with counts [E], kept [E], offsets [E+1], inv [T,K] (row or
    -1), src [N_kept] (token of each row), drop [T,K] uint8, n_dropped.
    """
    idx = np.asarray(idx)
    T, K = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    rank = np.zeros((T, K), dtype=np.int64)
    for t in range(T):                     # scan tokens in ascending order
        for k in range(K):
            e = int(idx[t, k])
            rank[t, k] = counts[e]
            counts[e] += 1
    kept = counts.copy() if C is None else np.minimum(counts, C)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)          # exclusive cumsum of kept counts
    inv = np.full((T, K), -1, dtype=np.int64)
    drop = np.zeros((T, K), dtype=np.uint8)
    src = np.zeros(int(offsets[E]), dtype=np.int64)
    for t in range(T):
        for k in range(K):
            e = int(idx[t, k])
            r = int(rank[t, k])
            if C is None or r < C:
                row = int(offsets[e]) + r
                inv[t, k] = row
                src[row] = t
            else:
                drop[t, k] = 1
    n_dropped = int(drop.sum())
    return dict(counts=counts, kept=kept, offsets=offsets, inv=inv, src=src,
                drop=drop, n_dropped=n_dropped)


# ---------------------------------------------------------------------------
# a5. Expert FFN
# ---------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a / (1 + exp(-a)), fp64."""
    return a / (1.0 + np.exp(-a))


def swiglu_ffn(X: np.ndarray, W1: np.ndarray, W3: np.ndarray, W2: np.ndarray,
               h_round=None) -> np.ndarray:
    """FFN(X) = (silu(X W1) * (X W3)) W2, row by row, in fp64.

    [P2] section 2 step 3 (each expert is an FFN); the SwiGLU form with W1 as
    the gate is the layer definition used here (READING).  ``h_round``, if
    given, is applied to H before the down projection (used to measure the
    floor that storing H in bf16 sets).
    """
    X = np.asarray(X, dtype=np.float64)
    H = silu(X @ np.asarray(W1, dtype=np.float64)) * (X @ np.asarray(W3, dtype=np.float64))
    if h_round is not None:
        H = h_round(H)
    return H @ np.asarray(W2, dtype=np.float64)


# ---------------------------------------------------------------------------
# a6. Combine
# ---------------------------------------------------------------------------

def combine(expert_out_rows: np.ndarray, inv: np.ndarray, w: np.ndarray, T: int,
            tokens=None) -> np.ndarray:
    """y[t] = sum over kept slots k of w[t,k] * Y[inv[t,k]], k = 0..K-1.

    [P2] section 2 step 4 and section 2.3 (weighted sum that restores token
    order); section 2.2 (an unselected or dropped expert contributes 0).
    READING: a dropped slot adds nothing and the other weights are not
    renormalised; a token with all slots dropped gets y = 0.
    ``tokens`` (bool mask [T]) limits the output to those tokens; other rows
    are NaN.
    """
    Y = np.asarray(expert_out_rows, dtype=np.float64)
    D = Y.shape[1]
    K = inv.shape[1]
    y = np.full((T, D), np.nan)
    for t in range(T):
        if tokens is not None and not tokens[t]:
            continue
        acc = np.zeros(D, dtype=np.float64)
        for k in range(K):
            r = int(inv[t, k])
            if r >= 0:
                acc = acc + float(w[t, k]) * Y[r]
        y[t] = acc
    return y


# ---------------------------------------------------------------------------
# a7. Aux-free bias update
# ---------------------------------------------------------------------------

def bias_update(bias32: np.ndarray, counts: np.ndarray, T: int, K: int, alpha: float) -> np.ndarray:
    """One aux-free balancing step, in fp32.

    [P3] section 1.2: an expert above the target load gets b -= alpha, one
    below gets b += alpha, one at the target is unchanged.
    READING: target = T*K/E, compared exactly as cnt*E vs T*K in integers;
    the load is the pre-drop selection count; b is fp32 and alpha is
    fl32(alpha), one fp32 add per step.
    """
    b = np.asarray(bias32, dtype=np.float32).copy()
    E = b.shape[0]
    a = np.float32(alpha)
    for e in range(E):
        lhs = int(counts[e]) * E
        rhs = T * K
        if lhs > rhs:
            b[e] = np.float32(b[e] - a)
        elif lhs < rhs:
            b[e] = np.float32(b[e] + a)
    return b


# ---------------------------------------------------------------------------
# The whole layer
# ---------------------------------------------------------------------------

def moe_layer(x, Wr, W1, W3, W2, K, capacity_factor=0.0, bias32=None, alpha=0.0,
              logits32=None, tokens=None, h_round=None):
    """The layer forward pass: steps a1..a7 in the pages' order.

    [P1] section 2 (route, dispatch, expert compute, aggregate back);
    [P2] sections 2, 2.1-2.3, 3.1, 1.2; [P3] sections 1, 1.2.

    x [T,d], Wr [d,E], W1/W3 [E,d,f], W2 [E,f,d] (arrays of bf16-rounded
    values, any float dtype); bias32 fp32 [E] or None.

    Routing decides in fp32: the fp64 logits are rounded to fp32 (unless
    ``logits32`` is given) and selection is done on fl32(l + b).
    ``tokens`` restricts the FFN/combine to those token ids (routing, counts
    and capacity still use all T tokens); y rows of other tokens are NaN.

    Returns a dict with logits (fp64), idx, w, counts, f, P, aux, P_topk,
    aux_topk, z_loss, dispatch
    fields, y_perm (expert-grouped FFN rows), y [T,d] fp64 and the updated
    bias.
    """
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape
    E = np.asarray(Wr).shape[1]
    l64 = router_logits(x, Wr)                              # a1 (unbiased)
    l32 = l64.astype(np.float32) if logits32 is None else np.asarray(logits32, np.float32)
    idx, w, _ = route_from_logits_f32(l32, K, bias32)       # a2
    probs = softmax_rows(l64)                               # a3 (unbiased)
    cnt = expert_counts(idx, E)
    f, P, aux = load_stats(cnt, probs, T, K)
    P_topk, aux_topk = topk_load_stats(cnt, idx, w, T, K)
    z_loss = router_z_loss(l64)
    C = capacity(T, K, E, capacity_factor)                  # a4
    disp = dispatch(idx, E, C)
    want = np.ones(T, dtype=bool)
    if tokens is not None:
        want[:] = False
        want[np.asarray(tokens, dtype=np.int64)] = True
    off, src = disp["offsets"], disp["src"]
    Yp = np.full((int(off[E]), d), np.nan)                  # a5: per expert group
    for e in range(E):
        rows = [r for r in range(int(off[e]), int(off[e + 1])) if want[int(src[r])]]
        if rows:
            Yp[rows] = swiglu_ffn(x[src[rows]], np.asarray(W1[e]), np.asarray(W3[e]),
                                  np.asarray(W2[e]), h_round)
    y = combine(Yp, disp["inv"], w, T, tokens=want)         # a6
    new_bias = None
    if bias32 is not None:
        new_bias = bias_update(bias32, cnt, T, K, alpha)    # a7
    out = dict(logits=l64, logits32=l32, idx=idx, w=w, counts=cnt, f=f, P=P, aux=aux, P_topk=P_topk,
               aux_topk=aux_topk, z_loss=z_loss,
               capacity=C, y=y, y_perm=Yp, bias=new_bias)
    out.update({k: v for k, v in disp.items() if k != "counts"})
    return out


# ---------------------------------------------------------------------------
# Offloaded experts: group-wise INT4 storage
# ---------------------------------------------------------------------------

INT4_GROUP = 64


def int4_quantize(W: np.ndarray, group: int = INT4_GROUP):
    """Group-wise symmetric 4-bit quantization of one expert matrix.

    [P3] section 3.2 (experts offloaded to CPU memory are stored group-wise
    quantized to INT4 to cut the transfer volume).
    READING (the page gives no scheme): W is [K_red, N] with the reduction
    axis first (W1, W3: [d_model, d_ff]; W2: [d_ff, d_model]); a group is
    `group` consecutive elements along the reduction axis for one column.
    Per group, in fp32: s = fl32(amax / 7) with amax = max |w| (w the fp32
    value of each weight), q = clamp(round_half_even(fl32(w / s)), -8, 7);
    an all-zero group has s = 0 and q = 0.  The divisions are correctly
    rounded fp32 divisions, so the codes are fixed bit for bit.

    Returns (q int8 [K_red, N], s float32 [K_red / group, N]).
    """
    w = np.asarray(W, dtype=np.float32)
    Kr, N = w.shape
    if Kr % group != 0:
        raise ValueError("the reduction length must be a multiple of the group")
    g = w.reshape(Kr // group, group, N)
    amax = np.max(np.abs(g), axis=1)                                  # [Kr/group, N] fp32
    s = (amax / np.float32(7.0)).astype(np.float32)                   # fp32 division
    safe = np.where(s > 0, s, np.float32(1.0))[:, None, :]
    r = (g / safe).astype(np.float32)                                 # fp32 division per weight
    q = np.clip(np.rint(r), -8, 7).astype(np.int8)                    # rint: ties to even
    q = np.where((s > 0)[:, None, :], q, np.int8(0))
    return q.reshape(Kr, N), s


def int4_dequantize(q: np.ndarray, s: np.ndarray, group: int = INT4_GROUP) -> np.ndarray:
    """w' = bf16(fl32(q * s)): the fp32 product rounded to bf16 (nearest
    even), widened to fp64.  The weight value the expert GEMM then uses."""
    q = np.asarray(q)
    Kr, N = q.shape
    srep = np.repeat(np.asarray(s, dtype=np.float32), group, axis=0)  # [Kr, N]
    prod = (q.astype(np.float32) * srep).astype(np.float32)
    return bf16_round(prod)


def lru_expert_cache(needed_per_step, n_slots: int, prefetch_per_step=None):
    """The LRU expert cache of [P3] section 3.2, step by step.

    [P3] section 3.2: keep the frequently used experts in a cache in GPU
    memory (LRU), and load the experts predicted for the next batch ahead of
    time.  READING (the page gives no algorithm):
      - before step t's expert computation every needed expert is resident;
        a hit refreshes its slot's last use to t;
      - misses, in ascending expert order, each take the slot with the
        smallest (last use, slot index) among the slots that hold no expert
        needed at step t; an empty slot has last use -1;
      - after step t, the experts of prefetch_per_step[t] (the prediction for
        step t + 1, in order) that are not resident are loaded the same way,
        into slots holding no expert used at step t, with last use t;
      - a step needing more experts than there are slots is an error.
    Returns one dict per step: hits (resident before the step and not loaded
    by the previous step's prefetch), prefetch_hits (loaded by that
    prefetch), misses (loaded on demand) as sorted expert lists, loads and
    prefetch_loads as [(expert, slot)], and slot_of {expert: slot} after the
    step's demand loads.
    """
    expert_of = [-1] * n_slots
    last_use = [-1] * n_slots
    slot_of = {}
    prefetched = set()
    out = []
    for t, needed in enumerate(needed_per_step):
        need = sorted(set(int(e) for e in needed))
        if len(need) > n_slots:
            raise ValueError(f"step {t} needs {len(need)} experts, the cache has {n_slots} slots")
        hits = [e for e in need if e in slot_of and e not in prefetched]
        phits = [e for e in need if e in slot_of and e in prefetched]
        misses = [e for e in need if e not in slot_of]
        for e in need:
            if e in slot_of:
                last_use[slot_of[e]] = t
        loads = []
        needset = set(need)

        def take(t_use, protect):
            cands = [(last_use[sl], sl) for sl in range(n_slots) if expert_of[sl] not in protect]
            return min(cands)[1] if cands else None

        for e in misses:
            sl = take(t, needset)
            old = expert_of[sl]
            if old >= 0:
                del slot_of[old]
            expert_of[sl] = e
            slot_of[e] = sl
            last_use[sl] = t
            loads.append((e, sl))
        snapshot = dict(slot_of)
        ploads = []
        prefetched = set()
        if prefetch_per_step is not None:
            for e in prefetch_per_step[t]:
                e = int(e)
                if e in slot_of:
                    continue
                sl = take(t, needset)
                if sl is None:
                    break
                old = expert_of[sl]
                if old >= 0:
                    del slot_of[old]
                expert_of[sl] = e
                slot_of[e] = sl
                last_use[sl] = t
                ploads.append((e, sl))
                prefetched.add(e)
        out.append(dict(hits=hits, prefetch_hits=phits, misses=misses, loads=loads, prefetch_loads=ploads,
                        slot_of=snapshot))
    return out


def routing_history_prediction(counts_per_step, width: int, beta: float = 0.75):
    """Experts predicted for the next step from the routing history.

    [P3] section 3.2 (predict from the routing history which experts the next
    batch needs, and load them ahead of time).  READING: a per-expert
    exponential moving average of the routed token counts, in fp32:
    c_e <- fl32(fl32(beta * c_e) + n_e(t)) with c_e = 0 before step 0; the
    prediction after step t is the `width` experts with the largest c_e
    (equal values: lower expert index first), in that order.
    """
    c = None
    b = np.float32(beta)
    preds = []
    for n in counts_per_step:
        n = np.asarray(n, dtype=np.float32)
        c = n.copy() if c is None else (b * c + n).astype(np.float32)
        order = np.argsort(-c, kind="stable")
        preds.append([int(e) for e in order[:width]])
    return preds


def dot_error_bound(x: np.ndarray, Wr: np.ndarray) -> np.ndarray:
    """Rigorous bound on |fp32-accumulated dot product - exact| per logit,
    before the final result is stored.

    Returns gamma_n * sum_i |x_i W_ie| with gamma_n = n u / (1 - n u),
    u = 2**-24: the accumulation error of an n-term sum of exact products in
    fp32 with round-to-nearest, for any summation order (Higham, Accuracy and
    Stability of Numerical Algorithms, section 3.1).  The term for rounding
    the exact logit itself to fp32 (u * |l|) is not included; callers that
    compare against an fp64 logit add it.
    """
    x = np.abs(np.asarray(x, dtype=np.float64))
    W = np.abs(np.asarray(Wr, dtype=np.float64))
    n = x.shape[1]
    u = 2.0 ** -24
    gamma = n * u / (1.0 - n * u)
    return gamma * (x @ W)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round to bf16 through fp32, and widen back to fp64.

    Two roundings, both to nearest with ties to even: fp64 -> fp32, then
    fp32 -> bf16.  This is the path of a value the kernels hold in fp32 (an
    fp32 accumulator stored as bf16).  It differs from a single fp64 -> bf16
    rounding only when the fp64 value lies within half an fp32 ulp of a bf16
    rounding midpoint (double rounding can then land on the even neighbour).
    """
    f = np.asarray(a, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    b = ((b + 0x7FFF + lsb) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)
