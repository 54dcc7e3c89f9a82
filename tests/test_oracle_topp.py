"""Pins of the oracle's top-p rule against things other than itself:
hand-derived fixtures, brute-force subset enumeration, monotonicity in p, and
the lognormal closed form for the kept fraction under flat N(0, s^2) scores."""

import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import top_p_set

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _brute_force(scores, p):
    """Minimum-cardinality subset with mass >= p; then maximum mass; then the
    lexicographically smallest sorted index tuple (lower indices win ties).
    Masses are summed with math.fsum (correctly rounded, order independent)."""
    s = np.asarray(scores, dtype=np.float64)
    n = len(s)
    w = np.exp(s - s.max())
    P = w / w.sum()
    if p >= 1.0:
        return list(range(n))
    for k in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), k):
            m = math.fsum(P[list(sub)])
            if m >= p:
                key = (-m, sub)
                if best is None or key < best:
                    best = key
        if best is not None:
            return list(best[1])
    return list(range(n))


def test_golden_two_token():
    d = json.load(open(os.path.join(GOLD, "topp_two_token.json")))
    for c in d["cases"]:
        assert list(top_p_set(np.array(d["scores"]), c["p"])) == c["kept"], c


def test_golden_ties():
    d = json.load(open(os.path.join(GOLD, "topp_ties.json")))
    for c in d["cases"]:
        assert list(top_p_set(np.array(c["scores"], dtype=float), c["p"])) == c["kept"], c


@pytest.mark.parametrize("seed", range(40))
def test_brute_force_random(seed):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 12))
    s = rng.normal(0, 2.0, size=n)
    if n > 3 and seed % 2 == 0:  # force exact ties
        s[rng.integers(0, n)] = s[0]
        s[rng.integers(0, n)] = s[1]
    for p in [0.05, 0.3, 0.5, 0.8, 0.9, 0.99, 1.0, float(rng.uniform(0.01, 0.999))]:
        assert list(top_p_set(s, p)) == _brute_force(s, p), (s, p)


@pytest.mark.parametrize("seed", range(10))
def test_brute_force_all_tied_blocks(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 11))
    s = rng.choice([-1.0, 0.0, 0.5], size=n)
    for p in np.linspace(0.02, 0.98, 25):
        assert list(top_p_set(s, float(p))) == _brute_force(s, float(p)), (s, p)


@pytest.mark.parametrize("seed", range(5))
def test_monotone_in_p(seed):
    rng = np.random.default_rng(seed)
    s = rng.normal(0, 1.5, size=3000)
    prev = None
    for p in np.linspace(0.01, 1.0, 60):
        kept = set(top_p_set(s, float(p)).tolist())
        if prev is not None:
            assert prev <= kept  # nested sets, hence monotone size
        prev = kept


@pytest.mark.parametrize("sigma,p", [(1.0, 0.95), (1.0, 0.8), (2.0, 0.95), (0.5, 0.9)])
def test_lognormal_kept_fraction(sigma, p):
    """Scores ~ N(0, sigma^2): mass above t is Phi(sigma - t/sigma), so keeping
    mass p keeps a fraction Phi(Phi^-1(p) - sigma) of the tokens."""
    from scipy.stats import norm
    rng = np.random.default_rng(7)
    n = 400_000
    s = rng.normal(0, sigma, size=n)
    frac = len(top_p_set(s, p)) / n
    expect = norm.cdf(norm.ppf(p) - sigma)
    assert abs(frac - expect) < 0.01, (frac, expect)


def test_p_one_keeps_all_and_empty():
    assert len(top_p_set(np.zeros(0), 0.5)) == 0
    assert list(top_p_set(np.array([3.0, -100.0, 0.0]), 1.0)) == [0, 1, 2]
