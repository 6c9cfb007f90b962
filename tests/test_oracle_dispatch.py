"""Pins of the oracle's capacity, keep-fraction, expert-choice and permutation.

Hand-worked fixtures (tests/golden/*_worked.json), the literal sequential
definition of the priority rule on small inputs, and invariants that hold
for any correct dispatch: counts sum to T*k minus drops, no expert exceeds
C, every expert holds exactly C rows in expert-choice mode, rows are the
inverse of the per-token map, x_perm rows are byte copies of x rows.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    return json.load(open(os.path.join(GOLD, name)))


def _check_layout(d: O.Dispatch, E: int):
    """Invariants of any dispatch: offsets scan kept, rows <-> map inverse."""
    assert d.offsets[0] == 0
    assert np.array_equal(np.diff(d.offsets), d.kept)
    R = int(d.offsets[-1])
    assert len(d.row_token) == R and len(d.row_gate) == R
    m = d.tok_rows
    rows = m[m >= 0]
    assert np.array_equal(np.sort(rows), np.arange(R))       # every row exactly once


def test_capacity_golden():
    g = _load("capacity_worked.json")
    d = O.dispatch_token_choice(np.array(g["topk_idx"]), np.array(g["topk_gate"], np.float32), None,
                                g["E"], capacity=g["capacity"])
    ex = g["expect"]
    assert d.counts.tolist() == ex["counts"]
    assert d.kept.tolist() == ex["kept"]
    assert d.offsets.tolist() == ex["offsets"]
    assert d.row_token.tolist() == ex["row_token"]
    assert d.row_gate.tolist() == ex["row_gate"]
    assert d.tok_rows.tolist() == ex["tok_rows"]
    assert d.n_dropped == ex["n_dropped"]


def test_capacity_matches_sequential_definition():
    """Literal rule: walk q = 0..T*k-1; keep if the expert has < C so far."""
    rng = np.random.default_rng(20)
    for (T, E, k, C) in [(64, 4, 2, 20), (100, 8, 3, 30), (257, 16, 2, 33), (50, 3, 3, 1)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        # skew: many tokens prefer expert 0 first
        idx[: T // 2, 0], idx[: T // 2, 1] = 0, idx[: T // 2, 1] % (E - 1) + 1
        gate = rng.random((T, k)).astype(np.float32)
        d = O.dispatch_token_choice(idx, gate, None, E, capacity=C)
        seen = np.zeros(E, int)
        keep = np.zeros((T, k), bool)
        for q in range(T * k):
            j, t = divmod(q, T)
            e = idx[t, j]
            keep[t, j] = seen[e] < C
            seen[e] += 1
        assert np.array_equal(d.tok_rows >= 0, keep)
        assert np.array_equal(d.counts, seen)
        assert np.array_equal(d.kept, np.minimum(seen, C))
        assert d.n_dropped == T * k - int(keep.sum())
        _check_layout(d, E)
        # row r of expert e is the (r - offsets[e])-th kept assignment of e in q order
        for e in range(E):
            qs = [q for q in range(T * k) if idx[q % T, q // T] == e and keep[q % T, q // T]]
            got = d.row_token[d.offsets[e]:d.offsets[e + 1]]
            assert got.tolist() == [q % T for q in qs]


def test_capacity_invariants_and_no_drop_limit():
    rng = np.random.default_rng(21)
    T, E, k = 4096, 16, 2
    l = rng.standard_normal((T, E)).astype(np.float32)
    p = O.softmax_det(l)
    idx, gate = O.topk_route(l, p, k)
    C = O.capacity_from_factor(T, E, k, 1.25)
    assert C == 640
    d = O.dispatch_token_choice(idx, gate, p, E, capacity=C)
    assert int(d.counts.sum()) == T * k
    assert int(d.kept.sum()) == T * k - d.n_dropped
    assert np.all(d.kept <= C)
    _check_layout(d, E)
    # every kept row's gate is the gate of its (t, j)
    t_, j_ = np.nonzero(d.tok_rows >= 0)
    assert np.array_equal(d.row_gate[d.tok_rows[t_, j_]], gate[t_, j_])
    assert np.array_equal(d.row_token[d.tok_rows[t_, j_]], t_)
    # capacity >= T*k never drops
    d2 = O.dispatch_token_choice(idx, gate, p, E, capacity=T * k)
    assert d2.n_dropped == 0 and np.all(d2.tok_rows >= 0)
    d3 = O.dispatch_token_choice(idx, gate, p, E, capacity=0)
    assert np.array_equal(d2.tok_rows, d3.tok_rows)


def test_all_tokens_on_one_expert():
    T, E, k, C = 50, 4, 1, 7
    idx = np.zeros((T, 1), np.int32)
    d = O.dispatch_token_choice(idx, np.ones((T, 1), np.float32), None, E, capacity=C)
    assert d.kept.tolist() == [C, 0, 0, 0]
    assert d.row_token.tolist() == list(range(C))          # the first C by priority
    assert d.n_dropped == T - C


def test_capacity_formula():
    # the two capacity-limited workloads: tiny fp32 and GShard-style
    assert O.capacity_from_factor(256, 8, 2, 1.25) == 80
    assert O.capacity_from_factor(4096, 16, 2, 1.25) == 640
    assert O.capacity_from_factor(100, 3, 2, 1.0) == math.ceil(200 / 3)
    assert O.capacity_from_factor(100, 3, 2, 0.0) == 0


def test_capacity_is_the_exact_ceiling():
    """For a factor num / 2^p (exact in binary) the capacity is the integer
    ceiling -(-(num * k * T) // (2^p * E)), with no rounding before it: e.g.
    1.1 * 2 * 500 / 10 = 110 exactly for the decimal 1.1, but the binary
    double 1.1 lies above it, so the exact ceiling is 111."""
    rng = np.random.default_rng(3)
    for _ in range(2000):
        p = int(rng.integers(0, 30))
        num = int(rng.integers(1, 1 << 24))
        T, E, k = int(rng.integers(1, 100000)), int(rng.integers(1, 300)), int(rng.integers(1, 9))
        want = -(-(num * k * T) // ((1 << p) * E))
        assert O.capacity_from_factor(T, E, k, num / (1 << p)) == want
    assert O.capacity_from_factor(500, 10, 2, 1.1) == 111
    assert O.capacity_from_factor(500, 10, 2, 1.25) == 125


def test_keep_fraction_golden():
    g = _load("keep_fraction_worked.json")
    idx = np.array(g["topk_idx"], np.int32)
    p = np.array(g["probs"], np.float32)
    gate = np.take_along_axis(p, idx, 1)
    d = O.dispatch_token_choice(idx, gate, p, g["E"], keep_num=g["keep_num"], keep_den=g["keep_den"])
    ex = g["expect"]
    for key in ("counts", "kept", "offsets", "row_token", "tok_rows"):
        assert getattr(d, key).tolist() == ex[key], key
    assert d.n_dropped == ex["n_dropped"]


def test_keep_fraction_invariants():
    rng = np.random.default_rng(22)
    T, E, k = 2000, 40, 6
    l = rng.standard_normal((T, E)).astype(np.float32)
    l[:, 3] += 1.0     # a hot expert
    p = O.softmax_det(l)
    idx, gate = O.topk_route(l, p, k, n_groups=8, topk_groups=3)
    d = O.dispatch_token_choice(idx, gate, p, E, keep_num=9, keep_den=10)
    assert np.array_equal(d.kept, (d.counts * 9 + 9) // 10)
    assert int(d.kept.sum()) == T * k - d.n_dropped
    _check_layout(d, E)
    for e in range(E):
        mask = idx == e
        toks = np.nonzero(mask.any(1))[0]
        kept_t = set(d.row_token[d.offsets[e]:d.offsets[e + 1]].tolist())
        pk = [(p[t, e], -t) for t in toks if t in kept_t]
        pd = [(p[t, e], -t) for t in toks if t not in kept_t]
        if pk and pd:
            assert min(pk) > max(pd)                       # kept beat dropped under (p, lower t)
        # rows stay in priority order (ascending t: each token meets e at most once)
        rt = d.row_token[d.offsets[e]:d.offsets[e + 1]]
        jt = np.array([np.nonzero(idx[t] == e)[0][0] * T + t for t in rt])
        assert np.all(np.diff(jt) > 0)


def test_keep_fraction_equal_affinity_keeps_lowest_tokens():
    T, E = 20, 2
    idx = np.zeros((T, 1), np.int32)
    p = np.full((T, E), 0.5, np.float32)
    d = O.dispatch_token_choice(idx, p[:, :1], p, E, keep_num=9, keep_den=10)
    assert d.row_token.tolist() == list(range(18))


def test_keep_all_equals_no_dropping():
    rng = np.random.default_rng(23)
    l = rng.standard_normal((300, 16)).astype(np.float32)
    p = O.softmax_det(l)
    idx, gate = O.topk_route(l, p, 4)
    a = O.dispatch_token_choice(idx, gate, p, 16, keep_num=1, keep_den=1)
    b = O.dispatch_token_choice(idx, gate, p, 16)
    assert a.n_dropped == 0 and np.array_equal(a.tok_rows, b.tok_rows)


def test_expert_choice_golden():
    g = _load("expert_choice_worked.json")
    d = O.dispatch_expert_choice(np.array(g["probs"], np.float32), g["C"])
    ex = g["expect"]
    for key in ("offsets", "row_token", "row_gate", "tok_rows"):
        assert getattr(d, key).tolist() == ex[key], key


def test_expert_choice_invariants():
    rng = np.random.default_rng(24)
    T, E = 1024, 64
    C = T * 6 // E
    l = (rng.standard_normal((T, E)) - 1.1 * np.log(np.arange(E) + 1.0)).astype(np.float32)
    p = O.softmax_det(l)
    d = O.dispatch_expert_choice(p, C)
    assert np.all(d.kept == C)
    _check_layout(d, E)
    for e in range(E):
        rt = d.row_token[e * C:(e + 1) * C]
        assert np.all(np.diff(rt) > 0)                     # ascending t
        assert np.array_equal(d.row_gate[e * C:(e + 1) * C], p[rt, e])
        sel = np.zeros(T, bool)
        sel[rt] = True
        ks = [(p[t, e], -t) for t in np.nonzero(sel)[0]]
        ns = [(p[t, e], -t) for t in np.nonzero(~sel)[0]]
        assert min(ks) > max(ns)
    # equal affinities: the lowest tokens win
    d2 = O.dispatch_expert_choice(np.full((10, 2), 0.5, np.float32), 3)
    assert d2.row_token.tolist() == [0, 1, 2, 0, 1, 2]


def test_permute_rows_are_byte_copies():
    rng = np.random.default_rng(25)
    x = rng.integers(0, 65535, size=(100, 32), dtype=np.uint16)      # bf16 bit patterns
    idx = rng.integers(0, 5, size=(100, 2)).astype(np.int32)
    idx[:, 1] = (idx[:, 0] + 1 + rng.integers(0, 4, 100)) % 5
    d = O.dispatch_token_choice(idx, np.ones((100, 2), np.float32), None, 5, capacity=30)
    xp = O.permute_rows(x, d)
    assert xp.dtype == np.uint16
    for r in range(len(d.row_token)):
        assert np.array_equal(xp[r], x[d.row_token[r]])
