"""Fit the router-weight skew of the skewed workloads on the oracle router.

TEST INFRASTRUCTURE (input construction).  Run once:

    python -m oracle.calibrate

It draws each workload's step-0 tokens and router weights from
``moe_layer_gemm_b200.synth`` and adjusts one skew parameter until the
oracle's pre-drop expert counts have the stated shape, then writes the
parameters to ``moe_layer_gemm_b200/workloads.json``.  The synth module only
reads those numbers; it never routes.

* mixtral_prefill: router column e is scaled by exp(gamma * g_e) (g_e seeded
  normals); gamma is bisected so that the coefficient of variation of the
  counts is 0.20.
* qwen_capacity: six seeded "hot" experts get a constant m added to their
  router column; with zero-mean tokens this raises the variance of their
  logits.  m is bisected so the hottest pre-drop count is 4x the mean load.
* deepseek_bias: per-expert column scales are fitted by the fixed-point
  iteration s_e <- s_e * (c_e / c_hat_e) ** 0.5 towards Zipf(1.1) counts over
  a seeded popularity order.  Zero-mean logits cannot select one expert for
  much more than half of the tokens, so the Zipf targets are capped at T/2
  and the excess is spread over the others in proportion to their targets.
"""
from __future__ import annotations

import json
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import moe_oracle as O  # noqa: E402
from moe_layer_gemm_b200 import synth  # noqa: E402


def _counts(x64, Wr_bf16, K, E):
    Wr = synth.bf16_to_f64(Wr_bf16)
    l32 = O.router_logits(x64, Wr).astype(np.float32)
    idx = O.topk_select(l32, K)
    return np.bincount(idx.reshape(-1), minlength=E)


def _cv(c):
    return float(np.std(c) / np.mean(c))


def fit_prefill(wl):
    x64 = synth.bf16_to_f64(synth.make_x(wl))
    g = synth.normal_f32(wl.E, wl.seed, synth.STREAM_SKEW).double()

    def counts(gamma):
        s = torch.exp(gamma * g).float()
        return _counts(x64, synth.make_router(wl, col_scale=s), wl.K, wl.E), s

    lo, hi = 0.0, 1.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        c, _ = counts(mid)
        if _cv(c) < 0.20:
            lo = mid
        else:
            hi = mid
    c, s = counts(0.5 * (lo + hi))
    return dict(gamma=0.5 * (lo + hi), scales=[float(v) for v in s], counts=c.tolist(), cv=_cv(c))


def fit_capacity(wl):
    x64 = synth.bf16_to_f64(synth.make_x(wl))
    hot = synth.distinct_choices(1, wl.E, 6, wl.seed, synth.STREAM_SKEW)[0].tolist()
    mean = wl.T * wl.K / wl.E

    def counts(m):
        shift = torch.zeros(wl.E)
        shift[hot] = m
        return _counts(x64, synth.make_router(wl, col_shift=shift), wl.K, wl.E)

    lo, hi = 0.0, 0.1
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if counts(mid).max() < 4 * mean:
            lo = mid
        else:
            hi = mid
    m = 0.5 * (lo + hi)
    c = counts(m)
    C = O.capacity(wl.T, wl.K, wl.E, wl.capacity_factor)
    return dict(hot=hot, shift=m, counts=c.tolist(), max_over_mean=float(c.max() / mean),
                capacity=C, dropped=int(np.maximum(c - C, 0).sum()))


def _zipf_targets(E, T, K, s, order):
    share = np.array([(r + 1.0) ** -s for r in range(E)])
    tgt = T * K * share / share.sum()
    cap = T / 2.0
    for _ in range(100):                 # cap and redistribute
        over = tgt > cap
        excess = float((tgt[over] - cap).sum())
        if excess <= 1e-9:
            break
        tgt[over] = cap
        free = ~over & (tgt < cap)
        tgt[free] += excess * tgt[free] / tgt[free].sum()
    out = np.zeros(E)
    out[order] = tgt                     # rank r -> expert order[r]
    return out


def fit_zipf(wl, iters=120):
    x64 = synth.bf16_to_f64(synth.make_x(wl))
    order = synth.distinct_choices(1, wl.E, wl.E, wl.seed, synth.STREAM_SKEW)[0].numpy()
    tgt = _zipf_targets(wl.E, wl.T, wl.K, 1.1, order)
    # The logits are linear in a column's scale, so the iteration scales the
    # unit-scale logits; the final scales are re-applied to the weights
    # before bf16 rounding and the reported counts come from those weights.
    base = O.router_logits(x64, synth.bf16_to_f64(synth.make_router(wl, col_scale=torch.ones(wl.E))))
    logs = np.zeros(wl.E)
    for it in range(iters):
        c = np.bincount(O.topk_select((base * np.exp(logs)).astype(np.float32), wl.K).reshape(-1),
                        minlength=wl.E)
        lr = 0.5 / (1.0 + it / 8.0)      # damped: the tail counts react sharply
        logs += np.clip(lr * (np.log(tgt) - np.log(np.maximum(c, 0.5))), -0.3, 0.3)
    s32 = [float(np.float32(v)) for v in np.exp(logs)]
    c = _counts(x64, synth.make_router(wl, col_scale=torch.tensor(s32, dtype=torch.float32)), wl.K, wl.E)
    ranks = np.empty(wl.E)
    ranks[order] = np.arange(1, wl.E + 1)
    ok = c > 0
    slope = float(np.polyfit(np.log(ranks[ok]), np.log(c[ok]), 1)[0])
    return dict(scales=s32, counts=c.tolist(), zipf_s=1.1, fitted_loglog_slope=slope,
                rel_l1_error=float(np.abs(c - tgt).sum() / (wl.T * wl.K)),
                max_count=int(c.max()), min_count=int(c.min()), experts_unused=int((c == 0).sum()))


def main():
    wls = synth.workloads()
    out = {}
    out["mixtral_prefill"] = fit_prefill(wls["mixtral_prefill"])
    print("mixtral_prefill", {k: v for k, v in out["mixtral_prefill"].items() if k != "scales"})
    out["qwen_capacity"] = fit_capacity(wls["qwen_capacity"])
    print("qwen_capacity", out["qwen_capacity"])
    out["deepseek_bias"] = fit_zipf(wls["deepseek_bias"])
    print("deepseek_bias", {k: v for k, v in out["deepseek_bias"].items() if k not in ("scales", "counts")})
    path = os.path.join(ROOT, "moe_layer_gemm_b200", "workloads.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
