"""Pins of the oracle's top-k sampler against facts that do not come from it: the order
statistics of a hand-written row, the extreme draws, and the closed-form distribution
(softmax over the kept logits at the temperature) reached by an even sweep of u.  Each
planted mistake (a forgotten temperature, one logit too many, the rank order reversed,
ties broken towards the higher index) must fail one of them."""
import numpy as np
import pytest
import torch

import oracle
from oracle import sampling as osm


def _sweep(sample, row, k, t, n=20000):
    counts = {}
    for j in range(n):
        tok = sample(row, k, t, (j + 0.5) / n)
        counts[tok] = counts.get(tok, 0) + 1
    return {tok: c / n for tok, c in counts.items()}


def _closed_form(row, k, t):
    """softmax(top-k logits / t), written with torch on float64 (not the oracle's arithmetic)."""
    v = torch.tensor(row, dtype=torch.float64)
    vals, idx = torch.topk(v, k)
    p = torch.softmax(vals / t, 0)
    return {int(i): float(q) for i, q in zip(idx, p)}


ROW = np.array([0.3, 2.0, -1.0, 1.5, 2.0, 0.9, -0.2, 1.1, 0.0, 1.7], dtype=np.float32)


def test_ranking_and_ties_lower_index_first():
    assert osm.top_k_ranked(ROW, 4) == [1, 4, 9, 3]
    assert osm.top_k_ranked(np.array([1, 3, 3, 2], dtype=np.float32), 2) == [1, 2]


def test_greedy_and_extreme_draws():
    assert oracle.sample_top_k(ROW, 1, 1.0, 0.99) == 1  # k = 1: argmax, lowest index of the max
    assert oracle.sample_top_k(ROW, 5, 0.8, 0.0) == 1  # u = 0: the largest
    assert oracle.sample_top_k(ROW, 5, 0.8, 1.0 - 2 ** -24) == 7  # u -> 1: the k-th largest
    # a tiny temperature puts all weight on the largest logits: here two equal ones (indices
    # 1 and 4), which share it evenly, the lower index first
    assert all(oracle.sample_top_k(ROW, 5, 1e-3, u) == 1 for u in (0.1, 0.3, 0.49))
    assert all(oracle.sample_top_k(ROW, 5, 1e-3, u) == 4 for u in (0.51, 0.7, 0.9))


@pytest.mark.parametrize("k, t", [(2, 1.0), (5, 0.7), (10, 2.0)])
def test_distribution_is_softmax_over_the_top_k(k, t):
    rng = np.random.default_rng(7)
    row = rng.normal(size=40).astype(np.float32)
    got = _sweep(oracle.sample_top_k, row, k, t)
    want = _closed_form(row, k, t)
    assert set(got) == set(want)
    for tok, p in want.items():
        assert abs(got[tok] - p) <= 2e-4, (tok, got[tok], p)


def _no_temperature(row, k, t, u):
    return oracle.sample_top_k(row, k, 1.0, u)


def _one_too_many(row, k, t, u):
    return oracle.sample_top_k(row, k + 1, t, u)


def _reversed_ranks(row, k, t, u):
    ranked = osm.top_k_ranked(row, k)[::-1]
    w = np.array([np.exp((float(row[i]) - float(row[ranked[-1]])) / t) for i in ranked])
    c = np.cumsum(w)
    return ranked[int(np.searchsorted(c, u * c[-1], side="right"))]


def _ties_to_higher_index(row, k, t, u):
    flipped = row[::-1].copy()
    return len(row) - 1 - oracle.sample_top_k(flipped, k, t, u)


@pytest.mark.parametrize("mutant", [_no_temperature, _one_too_many, _reversed_ranks, _ties_to_higher_index])
def test_planted_mistakes_are_caught(mutant):
    failed = False
    try:
        test_ranking_and_ties_lower_index_first()
        assert mutant(ROW, 5, 0.8, 0.0) == 1
        assert mutant(ROW, 1, 1.0, 0.5) == 1 and mutant(ROW, 2, 1.0, 0.0) == 1
        rng = np.random.default_rng(7)
        row = rng.normal(size=40).astype(np.float32)
        got = _sweep(mutant, row, 5, 0.7, n=4000)
        want = _closed_form(row, 5, 0.7)
        assert set(got) == set(want)
        for tok, p in want.items():
            assert abs(got[tok] - p) <= 1e-3
    except AssertionError:
        failed = True
    assert failed, f"{mutant.__name__} was not caught"


def test_boundary_margin_locates_the_running_sums():
    # u * total exactly on the first boundary: margin 0; halfway between: half a weight
    row = np.array([0.0, 0.0], dtype=np.float32)  # two equal weights: boundaries at 1/2 and 1
    assert osm.boundary_margin(row, 2, 1.0, 0.5) == 0.0
    assert abs(osm.boundary_margin(row, 2, 1.0, 0.25) - 0.25) < 1e-12
