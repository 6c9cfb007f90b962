"""Pins of the oracle's routing variants: DeepSeek-V3's bias routing and bias
update, load-aware top-k, GShard local groups.

* Worked examples built by hand from the pages' statements (golden/).
* Brute force: every k-subset of tiny inputs, keys formed by the stated
  rule, the best subset picked by enumeration.
* Special cases that reduce to plain top-k (zero bias, alpha = 0, full
  utilisation) and closed forms (a dominant bias forces an expert in).
* Local groups against an independent formulation: dispatching each group
  as its own batch and concatenating the rows group by group.
"""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _best_subset(keys, k):
    """k experts with the largest (key, -index), by enumeration, best first."""
    best = None
    for sub in itertools.combinations(range(len(keys)), k):
        ks = sorted(((float(keys[e]), -e) for e in sub), reverse=True)
        if best is None or ks > best:
            best = ks
    return [-e for (_, e) in best]


def _random_case(seed, T=48, E=6):
    rng = np.random.default_rng(seed)
    logits = (rng.integers(-8, 9, size=(T, E)) / 4.0).astype(F32)   # coarse grid: many ties
    probs = O.softmax_det(logits)
    return rng, logits, probs


def test_bias_routing_golden():
    g = json.load(open(os.path.join(GOLD, "bias_routing_worked.json")))
    p = np.asarray(g["probs"], F32)
    logits = np.log(p).astype(F32)
    idx, gate = O.topk_route(logits, p, g["k"], rule="bias", state=np.asarray(g["bias"], F32))
    assert idx.tolist() == g["expect_idx"]
    assert gate.tolist() == g["expect_gate"]
    u = g["update"]
    b2 = O.bias_update(u["counts"], g["bias"], u["T"], u["k"], u["gamma"])
    assert b2.tolist() == u["expect_bias"]


@pytest.mark.parametrize("seed", range(4))
def test_bias_rule_brute_force(seed):
    """Keys s + b with s = p; gates = the chosen keys."""
    rng, logits, probs = _random_case(seed)
    T, E = probs.shape
    b = (rng.integers(-24, 25, size=E) / 64.0).astype(F32)         # same scale as p
    k = 2
    idx, gate = O.topk_route(logits, probs, k, rule="bias", state=b)
    for t in range(T):
        keys = [F32(probs[t, e]) + F32(b[e]) for e in range(E)]     # fp32 sum of two fp32
        want = _best_subset(keys, k)
        assert idx[t].tolist() == want
        assert np.array_equal(gate[t], np.asarray([keys[e] for e in want], F32))


@pytest.mark.parametrize("seed", range(4))
def test_load_rule_brute_force(seed):
    """Keys g + alpha * (1 - u) on the logits; gates = p."""
    rng, logits, probs = _random_case(seed)
    T, E = probs.shape
    u = (rng.integers(0, 9, size=E) / 8.0).astype(F32)
    alpha = 1.5
    k = 3
    idx, gate = O.topk_route(logits, probs, k, rule="load", state=u, alpha=alpha)
    for t in range(T):
        keys = [float(logits[t, e]) + alpha * (1.0 - float(u[e])) for e in range(E)]  # exact here
        want = _best_subset(keys, k)
        assert idx[t].tolist() == want
        assert np.array_equal(gate[t], probs[t, want])


def test_variants_reduce_to_plain_topk():
    _, logits, probs = _random_case(7, T=64, E=8)
    idx0, gate0 = O.topk_route(logits, probs, 2)
    # alpha = 0, or every expert fully utilised: the load term vanishes exactly
    for u, a in ((np.linspace(0, 1, 8).astype(F32), 0.0), (np.ones(8, F32), 3.0)):
        idx, gate = O.topk_route(logits, probs, 2, rule="load", state=u, alpha=a)
        assert np.array_equal(idx, idx0) and np.array_equal(gate, gate0)
    # zero bias: keys are p, which orders the experts as the logits do
    # (ties aside: this grid has no two logits of a token closer than 1/4)
    rng = np.random.default_rng(3)
    l = (rng.permuted(np.tile(np.arange(8), (32, 1)), axis=1) / 4.0).astype(F32)
    p = O.softmax_det(l)
    idx0, gate0 = O.topk_route(l, p, 3)
    idx, gate = O.topk_route(l, p, 3, rule="bias", state=np.zeros(8, F32))
    assert np.array_equal(idx, idx0) and np.array_equal(gate, gate0)


def test_dominant_bias_forces_and_excludes():
    _, logits, probs = _random_case(11, T=40, E=6)
    b = np.zeros(6, F32)
    b[4], b[1] = 2.0, -2.0
    idx, gate = O.topk_route(logits, probs, 2, rule="bias", state=b)
    assert np.all(idx[:, 0] == 4)                       # p + 2 beats every p <= 1
    assert not np.any(idx == 1)                         # p - 2 < 0 loses to every p >= 0
    assert np.array_equal(gate[:, 0], (probs[:, 4] + F32(2.0)).astype(F32))


def test_bias_update_moves_toward_balance():
    rng = np.random.default_rng(5)
    E, T, k = 16, 256, 2
    counts = rng.multinomial(T * k, np.ones(E) / E)
    b = (rng.integers(-64, 65, size=E) / 1024.0).astype(F32)
    gamma = 2.0 ** -10                                 # exact steps on this grid
    b2 = O.bias_update(counts, b, T, k, gamma)
    mean = T * k / E
    for e in range(E):
        if counts[e] > mean:
            assert b2[e] == b[e] - F32(gamma)
        elif counts[e] < mean:
            assert b2[e] == b[e] + F32(gamma)
        else:
            assert b2[e] == b[e]
    # a non-dyadic step: one fp32 rounding of b -/+ fp32(gamma)
    b3 = O.bias_update(counts, b, T, k, 0.001)
    d = np.abs(b3.astype(np.float64) - b.astype(np.float64))
    moved = counts * E != T * k
    half_ulp = np.spacing(np.abs(b3[moved])).astype(np.float64) / 2
    assert np.all(np.abs(d[moved] - float(F32(0.001))) <= half_ulp)


def test_local_groups_golden():
    g = json.load(open(os.path.join(GOLD, "local_groups_worked.json")))
    d = O.dispatch_token_choice(np.asarray(g["topk_idx"], np.int32), np.asarray(g["topk_gate"], F32),
                                None, g["E"], g["capacity"], local_groups=g["G"])
    e = g["expect"]
    assert d.counts.tolist() == e["counts"]
    assert d.kept.tolist() == e["kept"]
    assert d.offsets.tolist() == e["offsets"]
    assert d.row_token.tolist() == e["row_token"]
    assert d.row_gate.tolist() == e["row_gate"]
    assert d.tok_rows.tolist() == e["tok_rows"]
    assert d.n_dropped == e["n_dropped"]


def test_group_capacity_closed_form():
    """Per-group capacity 2N/(G*E) for top-2 at capacity factor 1."""
    for N, G, E in ((4096, 4, 16), (1024, 8, 8), (960, 3, 10)):
        assert O.capacity_from_factor(N // G, E, 2, 1.0) == 2 * N // (G * E)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_local_groups_are_independent_batches(G):
    """Dispatch with G groups == each group dispatched as its own batch, rows
    concatenated group by group inside every expert."""
    rng = np.random.default_rng(G)
    T, E, k, C = 64, 5, 2, 4
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, k)).astype(F32)
    d = O.dispatch_token_choice(idx, gate, None, E, C, local_groups=G)
    Tg = T // G
    parts = [O.dispatch_token_choice(idx[g * Tg:(g + 1) * Tg], gate[g * Tg:(g + 1) * Tg], None, E, C)
             for g in range(G)]
    assert d.counts.tolist() == np.sum([p.counts for p in parts], axis=0).tolist()
    assert d.kept.tolist() == np.sum([p.kept for p in parts], axis=0).tolist()
    assert d.n_dropped == sum(p.n_dropped for p in parts)
    for e in range(E):
        rows = slice(d.offsets[e], d.offsets[e + 1])
        want_tok = np.concatenate([p.row_token[p.offsets[e]:p.offsets[e + 1]] + g * Tg
                                   for g, p in enumerate(parts)])
        want_gate = np.concatenate([p.row_gate[p.offsets[e]:p.offsets[e + 1]] for p in parts])
        assert d.row_token[rows].tolist() == want_tok.tolist()
        assert np.array_equal(d.row_gate[rows], want_gate)
    # tok_rows is the inverse of row_token
    for t in range(T):
        for j in range(k):
            r = d.tok_rows[t, j]
            if r >= 0:
                assert d.row_token[r] == t
