"""Pins of the oracle's top-k and group-limited selection.

Brute force: enumerate every k-subset (and every group subset) on tiny
inputs whose logits sit on a coarse grid so that ties are frequent, and pick
the best under the stated rule; the oracle must agree exactly.
"""
import itertools
import json
import os

import numpy as np

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _best_subset(l, k, allowed):
    """The k experts whose (logit, -index) keys are largest, by enumeration.

    Among all k-subsets of the allowed experts pick the one whose keys,
    sorted descending, are lexicographically largest; return it in that
    descending order.
    """
    best = None
    for sub in itertools.combinations(allowed, k):
        keys = sorted(((float(l[e]), -e) for e in sub), reverse=True)
        if best is None or keys > best:
            best = keys
    return [-e for (_, e) in best]


def _best_groups(l, n_groups, topk_groups):
    E = len(l)
    gsz = E // n_groups
    score = [max(float(v) for v in l[g * gsz:(g + 1) * gsz]) for g in range(n_groups)]
    best = None
    for sub in itertools.combinations(range(n_groups), topk_groups):
        keys = sorted(((score[g], -g) for g in sub), reverse=True)
        if best is None or keys > best:
            best = keys
    groups = [-g for (_, g) in best]
    return sorted(e for g in groups for e in range(g * gsz, (g + 1) * gsz))


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(10)
    for E in (1, 2, 3, 5, 8):
        for k in range(1, E + 1):
            l = (rng.integers(-8, 9, size=(64, E)) / 4.0).astype(np.float32)
            p = O.softmax_det(l)
            idx, gate = O.topk_route(l, p, k)
            for t in range(64):
                assert list(idx[t]) == _best_subset(l[t], k, list(range(E))), (E, k, t)
                assert np.array_equal(gate[t], p[t, idx[t]])


def test_group_limited_brute_force():
    rng = np.random.default_rng(11)
    for (E, n_groups, topk_groups, k) in [(8, 4, 2, 3), (8, 8, 3, 3), (6, 3, 1, 2), (12, 4, 3, 5), (8, 2, 1, 4)]:
        l = (rng.integers(-4, 5, size=(128, E)) / 4.0).astype(np.float32)
        p = O.softmax_det(l)
        idx, _ = O.topk_route(l, p, k, n_groups, topk_groups)
        for t in range(128):
            allowed = _best_groups(l[t], n_groups, topk_groups)
            assert list(idx[t]) == _best_subset(l[t], k, allowed), (E, n_groups, topk_groups, t)


def test_all_groups_reduces_to_plain_topk():
    rng = np.random.default_rng(12)
    l = (rng.standard_normal((300, 160))).astype(np.float32)
    p = O.softmax_det(l)
    a, ga = O.topk_route(l, p, 6, n_groups=8, topk_groups=8)
    b, gb = O.topk_route(l, p, 6)
    assert np.array_equal(a, b) and np.array_equal(ga, gb)


def test_topk_golden():
    g = json.load(open(os.path.join(GOLD, "gating_worked.json")))
    for case in g["topk_cases"]:
        l = np.array([case["logits"]], np.float32)
        p = O.softmax_det(l)
        ng, tg = case.get("n_groups", 0), case.get("topk_groups", 0)
        idx, _ = O.topk_route(l, p, case["k"], ng, tg)
        assert list(idx[0]) == case["idx"], case["why"]
        if "idx_no_groups" in case:
            idx2, _ = O.topk_route(l, p, case["k"])
            assert list(idx2[0]) == case["idx_no_groups"]


def test_renormalized_gates_sum_to_one():
    rng = np.random.default_rng(13)
    l = rng.standard_normal((500, 8)).astype(np.float32)
    p = O.softmax_det(l)
    idx, gate = O.topk_route(l, p, 2, renormalize=True)
    assert np.all(np.abs(gate.astype(np.float64).sum(1) - 1.0) <= 4 * 2.0 ** -24)
    # the ratio of the two gates is the ratio of their probabilities
    r = gate[:, 0].astype(np.float64) / gate[:, 1]
    rp = np.take_along_axis(p, idx, 1).astype(np.float64)
    assert np.allclose(r, rp[:, 0] / rp[:, 1], rtol=1e-6)
