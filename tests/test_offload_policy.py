"""The expert cache's policy on the host: the oracle pinned to a hand-traced
fixture, and the library's ExpertCache / HistoryPredictor against the oracle
on random routing traces, decision for decision."""
import json
import os

import numpy as np
import pytest

from moe_layer_gemm_b200.offload import ExpertCache, HistoryPredictor
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lru_cache_trace.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _pairs(x):
    return [tuple(p) for p in x]


def test_oracle_lru_matches_hand_trace():
    g = _golden()["demand"]
    out = O.lru_expert_cache(g["needed"], g["n_slots"])
    assert [_pairs(o["loads"]) for o in out] == [_pairs(x) for x in g["loads"]]
    assert [o["hits"] for o in out] == g["hits"]
    assert out[-1]["slot_of"] == {int(k): v for k, v in g["final_slot_of"].items()}


def test_oracle_lru_prefetch_matches_hand_trace():
    g = _golden()["prefetch"]
    out = O.lru_expert_cache(g["needed"], g["n_slots"], g["prefetch"])
    assert [_pairs(o["prefetch_loads"]) for o in out] == [_pairs(x) for x in g["prefetch_loads"]]
    assert [_pairs(o["loads"]) for o in out] == [_pairs(x) for x in g["loads"]]
    assert [o["prefetch_hits"] for o in out] == g["prefetch_hits"]
    assert [o["misses"] for o in out] == g["misses"]


def test_oracle_prediction_matches_hand_trace():
    g = _golden()["predictor"]
    assert O.routing_history_prediction(g["counts"], g["width"], g["beta"]) == g["predicted"]


def test_oracle_lru_rejects_a_step_larger_than_the_cache():
    with pytest.raises(ValueError):
        O.lru_expert_cache([[0, 1, 2]], 2)


@pytest.mark.parametrize("E,slots,width,seed", [(16, 6, 0, 1), (64, 24, 8, 2), (256, 96, 32, 3), (8, 8, 4, 4)])
def test_library_policy_matches_oracle_on_random_traces(E, slots, width, seed):
    rng = np.random.default_rng(seed)
    pop = (np.arange(E) + 1.0) ** -1.1          # Zipf-like popularity
    pop /= pop.sum()
    needed, counts = [], []
    for t in range(40):
        n = rng.multinomial(rng.integers(1, 3 * slots), pop)
        n[rng.permutation(E)[: max(0, int((n > 0).sum()) - slots)]] = 0   # at most `slots` experts a step
        nz = [int(e) for e in np.nonzero(n)[0]][:slots]
        keep = np.zeros(E, np.int64)
        keep[nz] = n[nz]
        needed.append(nz)
        counts.append(keep)
    preds = O.routing_history_prediction(counts, width) if width else None
    ref = O.lru_expert_cache(needed, slots, preds)
    cache = ExpertCache(slots)
    pred = HistoryPredictor(E, width) if width else None
    for t in range(len(needed)):
        hits, phits, misses, loads = cache.plan(needed[t])
        assert (hits, phits, misses) == (ref[t]["hits"], ref[t]["prefetch_hits"], ref[t]["misses"]), t
        assert loads == ref[t]["loads"], t
        assert {e: s for e, s in cache.where.items()} == ref[t]["slot_of"], t
        if pred is not None:
            p = pred.update(counts[t])
            assert p == preds[t], t
            assert cache.plan_prefetch(p) == ref[t]["prefetch_loads"], t
