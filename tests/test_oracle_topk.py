"""Pins of the oracle's static top-k rule (the pages' fixed-budget baseline,
atlas.scime.ai summary, "Baselines: static top-k") against things other than
itself: a hand-worked fixture with ties, brute-force subset enumeration, and
its relation to top-p (both keep a prefix of the same (score desc, index asc)
order, so top-k with k = |top-p set| is that set)."""

import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleCache, top_k_set, top_p_set
from synth import LayerShape

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _brute_force(scores, k):
    """Among all k-subsets: maximum score sum, then the lexicographically
    smallest sorted index tuple (lower indices win ties)."""
    s = np.asarray(scores, dtype=np.float64)
    n = len(s)
    k = min(k, n)
    best = None
    for sub in itertools.combinations(range(n), k):
        key = (-sum(sorted(s[list(sub)])), sub)  # sum in a fixed order: ties compare exactly
        if best is None or key < best:
            best = key
    return list(best[1])


def test_golden_ties():
    d = json.load(open(os.path.join(GOLD, "topk_ties.json")))
    for c in d["cases"]:
        assert list(top_k_set(np.array(d["scores"]), c["k"])) == c["kept"], c


@pytest.mark.parametrize("seed", range(30))
def test_brute_force_random(seed):
    rng = np.random.default_rng(2000 + seed)
    n = int(rng.integers(1, 11))
    s = np.round(rng.normal(0, 2.0, size=n), 1)  # rounding forces ties
    for k in range(1, n + 2):
        assert list(top_k_set(s, k)) == _brute_force(s, k), (s, k)


@pytest.mark.parametrize("seed", range(10))
def test_topk_of_topp_size_is_the_topp_set(seed):
    rng = np.random.default_rng(3000 + seed)
    s = rng.normal(0, 1.5, size=500)
    s[rng.integers(0, 500, 20)] = s[3]  # ties
    for p in (0.3, 0.8, 0.95):
        tp = top_p_set(s, p)
        assert np.array_equal(top_k_set(s, len(tp)), tp)


def test_layer_uses_topk_when_configured():
    """A decode step of a layer with top_k keeps exactly k tokens per retrieval
    q head: the k highest scores of the indexer (checked against a direct
    argsort of the scores)."""
    sh = LayerShape(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=32, n_sink=2, window=4,
                    top_p=0.9, retrieval=(0,), dtype="fp32", top_k=7)
    g = torch.Generator().manual_seed(4)
    L = 60
    k = torch.randn((1, L, 1, 32), generator=g)
    v = torch.randn((1, L, 1, 32), generator=g)
    q = torch.randn((1, 2, 32), generator=g)
    wq = torch.randn((1, 16, 32), generator=g) / 32 ** 0.5
    wk = torch.randn((1, 16, 32), generator=g) / 32 ** 0.5
    c = OracleCache(sh, L)
    c.append(k, v, [0], L, wk)
    _, topk, final = oracle.decode(c, q, [L], wq)
    for hq in range(2):
        s = (k[0, :, 0].double().numpy() @ wk[0].double().numpy().T) @ (wq[0].double().numpy() @ q[0, hq].double().numpy()) / 4
        want = np.sort(np.argsort(-s, kind="stable")[:7])
        assert list(topk[(0, hq)]) == list(want)
        assert set(final[(0, hq)]) == set(want) | set(oracle.sink_window_set(L - 1, 2, 4))
