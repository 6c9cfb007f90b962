"""Pins of the oracle's backward pass (gradients of L = sum(dy * y), routing
held fixed).

* Central finite differences of the float64 forward with the same selection
  (gates from the exact softmax) for every parameter kind, in each routing
  mode: capacity, renormalised SwiGLU with shared experts, keep-fraction
  with group limits, expert choice, DeepSeek-V3 bias routing, load-aware
  top-k, local groups.
* An independent autograd evaluation: the dense soft mixture (k = E, nothing
  dropped) written directly in torch float64, differentiated by torch.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

CASES = {
    "capacity_relu": dict(E=4, S=0, k=2, act="relu", capacity=4),
    "renorm_swiglu_shared": dict(E=4, S=1, k=2, act="swiglu", renormalize=True),
    "keepfrac_groups": dict(E=6, S=1, k=2, act="swiglu", keep_num=2, keep_den=3, n_groups=3,
                            topk_groups=2),
    "expert_choice": dict(E=4, S=1, k=2, act="swiglu", mode="ec", ec_capacity=5),
    "bias_rule": dict(E=4, S=1, k=2, act="swiglu", rule="bias"),
    "load_rule": dict(E=4, S=0, k=2, act="relu", rule="load", alpha=0.5),
    "local_groups": dict(E=4, S=0, k=2, act="relu", capacity=2, local_groups=2),
}


def _problem(seed, cfg, T=12, d=6, f=5, with_bias=True):
    rng = np.random.default_rng(seed)
    G = cfg.E + cfg.S
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((cfg.E, d)) * 0.7
    bias = rng.standard_normal(cfg.E) * 0.3 if with_bias else None
    w1 = rng.standard_normal((G, f, d)) * 0.5
    w3 = rng.standard_normal((G, f, d)) * 0.5 if cfg.act == "swiglu" else None
    w2 = rng.standard_normal((G, d, f)) * 0.5
    dy = rng.standard_normal((T, d))
    state = None
    if cfg.rule == "bias":
        state = (rng.standard_normal(cfg.E) * 0.05).astype(np.float32)
    elif cfg.rule == "load":
        state = rng.random(cfg.E).astype(np.float32)
    return x, wr, bias, w1, w3, w2, dy, state


def _loss(cfg, disp, idx, state, dy, x, wr, bias, w1, w3, w2):
    y = O.forward_fixed_selection(cfg, x, wr, bias, w1, w3, w2, disp, idx, state)
    return float(np.sum(dy * y))


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_finite_differences(name):
    cfg = O.OracleConfig(**CASES[name])
    x, wr, bias, w1, w3, w2, dy, state = _problem(1, cfg)
    logits32 = O.router_logits(x, wr, bias)
    _, idx, _, disp = O.route(cfg, logits32, state)
    g = O.backward(cfg, x, wr, bias, w1, w3, w2, dy, state)
    params = {"x": (x, g.dx), "wr": (wr, g.dw_router), "bias": (bias, g.dbias),
              "w1": (w1, g.dw1), "w2": (w2, g.dw2)}
    if w3 is not None:
        params["w3"] = (w3, g.dw3)
    rng = np.random.default_rng(2)
    h = 1e-6
    for pname, (arr, grad) in params.items():
        flat = arr.reshape(-1)
        picks = rng.choice(flat.size, size=min(flat.size, 24), replace=False)
        for i in picks:
            old = flat[i]
            vals = []
            for s in (+1, -1):
                flat[i] = old + s * h
                vals.append(_loss(cfg, disp, idx, state, dy, x, wr, bias, w1, w3, w2))
            flat[i] = old
            fd = (vals[0] - vals[1]) / (2 * h)
            an = grad.reshape(-1)[i]
            assert abs(fd - an) <= 1e-6 * (1 + abs(fd)), f"{name}: d{pname}[{i}] fd {fd} vs {an}"


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_dense_mixture_matches_torch_autograd(act):
    """k = E, no capacity: y = sum_e softmax(x W_r^T)_e FFN_e(x) + FFN_shared(x),
    written directly in torch float64 and differentiated by torch."""
    cfg = O.OracleConfig(E=3, S=1, k=3, act=act)
    x, wr, bias, w1, w3, w2, dy, state = _problem(5, cfg, with_bias=False)
    g = O.backward(cfg, x, wr, None, w1, w3, w2, dy)
    t = {n: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for n, v in (("x", x), ("wr", wr), ("w1", w1), ("w2", w2)) + ((("w3", w3),) if w3 is not None else ())}
    p = torch.softmax(t["x"] @ t["wr"].T, dim=1)

    def ffn(e):
        a = t["x"] @ t["w1"][e].T
        h = torch.relu(a) if act == "relu" else torch.nn.functional.silu(a) * (t["x"] @ t["w3"][e].T)
        return h @ t["w2"][e].T

    y = sum(p[:, e:e + 1] * ffn(e) for e in range(cfg.E)) + ffn(cfg.E)
    (y * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(g.dx, t["x"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g.dw_router, t["wr"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g.dw1, t["w1"].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g.dw2, t["w2"].grad.numpy(), rtol=1e-10, atol=1e-12)
    if act == "swiglu":
        np.testing.assert_allclose(g.dw3, t["w3"].grad.numpy(), rtol=1e-10, atol=1e-12)


def test_dropped_rows_get_no_gradient():
    """An expert whose every assignment overflowed receives zero weight
    gradient; tokens that lost an expert get no gradient from it."""
    cfg = O.OracleConfig(E=2, S=0, k=1, act="relu", capacity=1)
    x, wr, bias, w1, w3, w2, dy, _ = _problem(9, cfg, T=6, with_bias=False)
    bias = np.array([30.0, -30.0])                    # everyone picks expert 0; capacity keeps one
    g = O.backward(cfg, x, wr, bias, w1, None, w2, dy)
    assert np.all(g.dw1[1] == 0) and np.all(g.dw2[1] == 0)
    _, idx, _, disp = O.route(cfg, O.router_logits(x, wr, bias))
    kept_tok = disp.row_token.tolist()
    assert len(kept_tok) == 1
    for t in range(6):
        if t not in kept_tok:        # no kept row: no expert and no gate gradient reaches t
            assert np.all(g.dx[t] == 0.0)
