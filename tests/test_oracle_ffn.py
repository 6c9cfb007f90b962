"""Pins of the oracle's expert FFNs and combine against independent torch
float64 evaluations of the special cases the pages fix:

* k = E with no capacity limit is the dense soft mixture sum_e p_e FFN_e(x)
  ("MoE技术演进", Adaptive Mixtures of Local Experts);
* E = 1, k = 1 is a plain dense FFN (GShard section 3, FFN_e equation);
* shared experts alone give sum_s FFN_s(x) (DeepSeekMoE section 2);
* relabelling the experts (router rows and weights together) changes nothing.

The dense side never routes, permutes or gathers: it applies every expert to
every token with torch.nn.functional.linear.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_oracle as O


def _rand(rng, shape, std):
    return (rng.standard_normal(shape) * std).astype(np.float32)


def _dense_ffn(x, w1, w2, w3, act):
    x = torch.from_numpy(np.asarray(x, np.float64))
    g = F.linear(x, torch.from_numpy(np.asarray(w1, np.float64)))
    if act == "relu":
        h = F.relu(g)
    else:
        h = F.silu(g) * F.linear(x, torch.from_numpy(np.asarray(w3, np.float64)))
    return F.linear(h, torch.from_numpy(np.asarray(w2, np.float64))).numpy()


def _make(rng, T, d, E, S, f, act):
    x = _rand(rng, (T, d), 1.0)
    wr = _rand(rng, (E, d), d ** -0.5)
    w1 = _rand(rng, (E + S, f, d), d ** -0.5)
    w3 = _rand(rng, (E + S, f, d), d ** -0.5) if act == "swiglu" else None
    w2 = _rand(rng, (E + S, d, f), f ** -0.5)
    return x, wr, w1, w3, w2


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_k_equals_E_is_dense_soft_mixture(act):
    rng = np.random.default_rng(30)
    T, d, E, f = 40, 32, 6, 48
    x, wr, w1, w3, w2 = _make(rng, T, d, E, 0, f, act)
    cfg = O.OracleConfig(E=E, S=0, k=E, act=act)
    res = O.forward(cfg, x, wr, None, w1, w3, w2)
    p = torch.softmax(F.linear(torch.from_numpy(x).double(), torch.from_numpy(wr).double()), 1).numpy()
    ref = sum(p[:, e:e + 1] * _dense_ffn(x, w1[e], w2[e], None if w3 is None else w3[e], act) for e in range(E))
    # the oracle's gates are fp32 probabilities: relative error ~1e-6
    assert np.allclose(res.y, ref, rtol=1e-5, atol=1e-5 * np.abs(ref).max())


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_single_expert_is_dense_ffn(act):
    rng = np.random.default_rng(31)
    T, d, f = 25, 64, 96
    x, wr, w1, w3, w2 = _make(rng, T, d, 1, 0, f, act)
    cfg = O.OracleConfig(E=1, S=0, k=1, act=act)
    res = O.forward(cfg, x, wr, None, w1, w3, w2)
    assert np.all(res.probs == 1.0)
    ref = _dense_ffn(x, w1[0], w2[0], None if w3 is None else w3[0], act)
    assert np.allclose(res.y, ref, rtol=1e-12, atol=1e-12)


def test_shared_experts_alone():
    rng = np.random.default_rng(32)
    T, d, E, S, f = 30, 32, 4, 2, 40
    x, wr, w1, w3, w2 = _make(rng, T, d, E, S, f, "swiglu")
    # keep 0 of every expert's assignments: only the shared experts remain
    cfg = O.OracleConfig(E=E, S=S, k=2, act="swiglu", keep_num=0, keep_den=1)
    res = O.forward(cfg, x, wr, None, w1, w3, w2)
    assert res.dispatch.n_dropped == T * 2
    ref = sum(_dense_ffn(x, w1[E + s], w2[E + s], w3[E + s], "swiglu") for s in range(S))
    assert np.allclose(res.y, ref, rtol=1e-12, atol=1e-12)


def test_shared_term_independent_of_routing():
    rng = np.random.default_rng(33)
    T, d, E, S, f = 30, 32, 6, 2, 40
    x, wr, w1, w3, w2 = _make(rng, T, d, E, S, f, "swiglu")
    cfg = O.OracleConfig(E=E, S=S, k=2, act="swiglu")
    a = O.forward(cfg, x, wr, None, w1, w3, w2).y
    cfg0 = O.OracleConfig(E=E, S=0, k=2, act="swiglu")
    b = O.forward(cfg0, x, wr, None, w1[:E], w3[:E], w2[:E]).y
    shared = sum(_dense_ffn(x, w1[E + s], w2[E + s], w3[E + s], "swiglu") for s in range(S))
    assert np.allclose(a - b, shared, rtol=1e-10, atol=1e-12)


def test_topk_mixture_against_dense_masked_sum():
    """Routed top-k with capacity: y = sum over kept (t, e) of p * FFN_e(x_t),
    evaluated densely (every expert on every token) and masked."""
    rng = np.random.default_rng(34)
    T, d, E, k, f = 64, 32, 8, 2, 48
    x, wr, w1, w3, w2 = _make(rng, T, d, E, 0, f, "relu")
    C = O.capacity_from_factor(T, E, k, 1.0)
    cfg = O.OracleConfig(E=E, S=0, k=k, act="relu", capacity=C)
    res = O.forward(cfg, x, wr, None, w1, w3, w2)
    dense = np.stack([_dense_ffn(x, w1[e], w2[e], None, "relu") for e in range(E)])   # [E, T, d]
    ref = np.zeros((T, d))
    for t in range(T):
        for j in range(k):
            if res.dispatch.tok_rows[t, j] >= 0:
                e = res.topk_idx[t, j]
                ref[t] += float(res.probs[t, e]) * dense[e, t]
    assert np.allclose(res.y, ref, rtol=1e-12, atol=1e-12)
    assert res.dispatch.n_dropped > 0


def test_expert_choice_against_dense_masked_sum():
    rng = np.random.default_rng(35)
    T, d, E, S, f = 48, 32, 8, 1, 40
    x, wr, w1, w3, w2 = _make(rng, T, d, E, S, f, "swiglu")
    C = T * 2 // E
    cfg = O.OracleConfig(E=E, S=S, k=2, act="swiglu", mode="ec", ec_capacity=C)
    res = O.forward(cfg, x, wr, None, w1, w3, w2)
    dense = np.stack([_dense_ffn(x, w1[e], w2[e], w3[e], "swiglu") for e in range(E + S)])
    ref = dense[E].copy()
    for e in range(E):
        for t in res.dispatch.row_token[e * C:(e + 1) * C]:
            ref[t] += float(res.probs[t, e]) * dense[e, t]
    assert np.allclose(res.y, ref, rtol=1e-12, atol=1e-12)


def test_expert_relabelling_invariance():
    rng = np.random.default_rng(36)
    T, d, E, k, f = 50, 32, 8, 2, 40
    x, wr, w1, w3, w2 = _make(rng, T, d, E, 0, f, "swiglu")
    perm = rng.permutation(E)
    cfg = O.OracleConfig(E=E, S=0, k=k, act="swiglu", capacity=O.capacity_from_factor(T, E, k, 1.0))
    a = O.forward(cfg, x, wr, None, w1, w3, w2)
    b = O.forward(cfg, x, wr[perm], None, w1[perm], w3[perm], w2[perm])
    # same experts chosen and dropped, under the new labels
    assert np.array_equal(perm[b.topk_idx], a.topk_idx)
    assert np.array_equal(b.dispatch.tok_rows >= 0, a.dispatch.tok_rows >= 0)
    # the fp32 softmax denominator is summed in label order: gates move by ulps
    assert np.allclose(a.y, b.y, rtol=1e-5, atol=1e-6 * np.abs(a.y).max())


def test_sampled_tokens_match_full_forward():
    rng = np.random.default_rng(37)
    T, d, E, S, f = 80, 32, 8, 1, 40
    x, wr, w1, w3, w2 = _make(rng, T, d, E, S, f, "swiglu")
    cfg = O.OracleConfig(E=E, S=S, k=3, act="swiglu", keep_num=9, keep_den=10, n_groups=4, topk_groups=2)
    full = O.forward(cfg, x, wr, None, w1, w3, w2)
    toks = np.array([0, 7, 79, 33])
    part = O.forward(cfg, x, wr, None, w1, w3, w2, tokens=toks)
    # float64 BLAS blocks differently for different row counts
    assert np.allclose(part.y, full.y[toks], rtol=1e-12, atol=1e-14)
