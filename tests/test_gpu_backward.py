"""Backward pass on the GPU against the oracle's float64 backward (routing
held fixed): dx, dW_r, d(logit bias), dW1, dW3, dW2.

Inputs on the routing grid, so the GPU's forward routing equals the
oracle's bit for bit (checked through the counts); dy seeded N(0, 1) in
bf16.  The contractions take bf16 operands (x, dy, recomputed
pre-activations, dA / dU, transposed copies: each rounded once, 2^-9
relative) with fp32 accumulation, a chain of at most three such roundings,
and every gradient is a sum of terms of both signs whose cancellation
magnifies the relative error of single elements.  The rule, per slice of the
leading dimension (one token of dx, one expert of each weight gradient):
||g - g_ref|| <= 2e-2 ||g_ref|| and max |g - g_ref| <= 3e-2 max |g_ref|
(an element's error is measured against the slice's largest value: a
lightly loaded expert's gradient is a sum of a few outer products, heavy
tailed, and its largest elements carry the largest roundings).  With ReLU
the same 3e-2 element bound holds everywhere except where a mask can
legitimately differ: a pre-activation whose exact value lies within the
accumulation error of its fp32 recomputation (|a| <= K * 2^-22 * sum |x_i w_i|,
four fp32 roundings per added term) may come out on the other side of
zero, both correct, and the ReLU mask (the derivative is discontinuous
there) then takes or drops a whole term dh * x.  Only the elements such a
position feeds -- the row j of dW1_e, and the token's row of dx -- are held
to the looser 1e-1 max |g_ref|.  Slices, because experts differ in load,
so their gradients differ in scale by an order of magnitude or more, and
each slice carries its own rounding at its own scale.  An all-zero reference slice (an
expert without rows) must come out exactly zero.  The router's gradients are
sums over tokens of terms with both signs (dbias_e = sum_t dl[t, e], dW_r =
dl^T x) whose cancellation is data-dependent, so their bound is 3e-2 times
the root sum of squares of the summed terms (the reference's dl), the size
of the accumulated per-term rounding."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS
from oracle import moe_oracle as O
from tests.gpu_common import (SMALL, LazyExperts, gpu_inputs, oracle_config, state_np, to_f64,
                              to_np)

pytestmark = pytest.mark.gpu

TOL = 3e-2          # router gradients, times the root sum of squares of the summed terms
TOL_FRO = 2e-2      # per slice, relative Frobenius norm
TOL_MAX = 3e-2      # per slice, max error over the largest reference value
BF16_SMALL = [n for n, w in SMALL.items() if w.dtype == "bf16"]


TOL_MAX_MASK = 1e-1  # ReLU: elements fed by a pre-activation whose sign may differ


def _check(name, got, ref, loose=None):
    """Per slice of the leading dimension: relative Frobenius error within
    TOL_FRO, every element within TOL_MAX of the slice's largest value, or
    within TOL_MAX_MASK where `loose` (a boolean array of ref's shape) is set."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64).reshape(ref.shape)
    n = ref.shape[0]
    r2 = ref.reshape(n, -1)
    g2 = got.reshape(n, -1)
    rms = np.sqrt(np.mean(r2 ** 2, axis=1))
    top = np.abs(r2).max(axis=1)
    tol = np.full(r2.shape, TOL_MAX)
    if loose is not None:
        tol[np.asarray(loose).reshape(n, -1)] = TOL_MAX_MASK
    over = (np.abs(g2 - r2) / (tol * top[:, None] + 1e-300)).max(axis=1)   # > 1: out of bound
    err = np.abs(g2 - r2).max(axis=1)
    fro = np.sqrt(np.mean((g2 - r2) ** 2, axis=1))
    zero = rms == 0
    assert np.all(err[zero] == 0), f"{name}: nonzero gradient where the reference is zero"
    nz = np.flatnonzero(~zero)
    bad = nz[(fro[nz] > TOL_FRO * rms[nz]) | (over[nz] > 1.0)]
    if len(bad):
        i = bad[0]
        raise AssertionError(f"{name}[{i}]: rel. error {fro[i] / rms[i]:.3e}, max|err| / max|ref| "
                             f"{err[i] / top[i]:.3e}")


def _relu_ambiguous(w, x_np, w1, disp):
    """Where the sign of a ReLU pre-activation is within rounding: returns
    (rows_of_dw1 [E+S, f] bool, tokens [T] bool) of the elements it feeds."""
    xs = O.widen(x_np)
    K = xs.shape[1]
    amb_w = np.zeros((w.E + w.S, w.d_ff), dtype=bool)
    amb_t = np.zeros(w.T, dtype=bool)
    for e in range(w.E + w.S):
        if e < w.E:
            toks = disp.row_token[disp.offsets[e]:disp.offsets[e + 1]]
        else:
            toks = np.arange(w.T)
        if len(toks) == 0:
            continue
        we = O.widen(w1[e])
        a = xs[toks] @ we.T
        bound = K * 2.0 ** -22 * (np.abs(xs[toks]) @ np.abs(we).T)
        near = np.abs(a) <= bound
        amb_w[e] |= near.any(axis=0)
        amb_t[toks[near.any(axis=1)]] = True
    return amb_w, amb_t


def _backward_check(w, seed=21):
    inp = gpu_inputs(w, seed=seed, grid=True)
    cfg = api.config_from_workload(w)
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias,
                         route_state=inp.route_state)
    layer(inp.x)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    dy = torch.randn(w.T, w.d_model, generator=g, device="cuda").to(torch.bfloat16)
    grads = layer.backward(inp.x, dy)
    torch.cuda.synchronize()
    api.moe_check_device_errors(layer.ws)
    oc = oracle_config(w)
    x_np = to_np(inp.x)
    bias = None if inp.bias is None else to_np(inp.bias)
    st = state_np(inp)
    _, _, _, disp = O.route(oc, O.router_logits(x_np, to_np(inp.w_router), bias), st)
    assert np.array_equal(layer.counts.cpu().numpy(), disp.counts)      # same routing
    G = w.E + w.S
    w1 = [to_np(inp.w1[e]) for e in range(G)]
    w2 = [to_np(inp.w2[e]) for e in range(G)]
    w3 = [to_np(inp.w3[e]) for e in range(G)] if inp.w3 is not None else None
    ref = O.backward(oc, x_np, to_np(inp.w_router), bias, w1, w3, w2, to_f64(dy), st, disp)
    loose_w1 = loose_x = None
    if w.act == "relu":
        amb_w, amb_t = _relu_ambiguous(w, x_np, w1, disp)
        loose_w1 = np.broadcast_to(amb_w[:, :, None], ref.dw1.shape)
        loose_x = np.broadcast_to(amb_t[:, None], ref.dx.shape)
    _check("dx", to_f64(grads["dx"]), ref.dx, loose_x)
    dl = ref.dlogits
    xs = O.widen(x_np)
    rss_w = np.sqrt((dl ** 2).T @ (xs ** 2))             # [E, d]
    err_w = np.abs(to_f64(grads["dw_router"]) - ref.dw_router)
    assert np.all(err_w <= TOL * rss_w + 1e-12), \
        f"dw_router: worst err / rss {float((err_w / (rss_w + 1e-30)).max()):.3e}"
    if bias is not None:
        rss_b = np.sqrt((dl ** 2).sum(axis=0))
        err_b = np.abs(to_f64(grads["dbias"]) - ref.dbias)
        assert np.all(err_b <= TOL * rss_b + 1e-12), \
            f"dbias: worst err / rss {float((err_b / (rss_b + 1e-30)).max()):.3e}"
    _check("dw1", to_f64(grads["dw1"]), ref.dw1, loose_w1)
    _check("dw2", to_f64(grads["dw2"]), ref.dw2)
    if w3 is not None:
        _check("dw3", to_f64(grads["dw3"]), ref.dw3)


@pytest.mark.parametrize("name", BF16_SMALL)
def test_backward_small(name):
    _backward_check(SMALL[name])


def test_backward_expert_without_rows():
    """An expert that gets no row still gets its (zero) weight gradient."""
    w = replace(SMALL["gshard_s"], T=256, E=8, zipf_s=3.0, capacity_factor=0.0)
    _backward_check(w)


def test_backward_full_size_gshard():
    """The benchmark's GShard-shaped layer at full size."""
    _backward_check(WORKLOADS["gshard"])


def test_backward_is_deterministic():
    w = SMALL["pair_swiglu_s"]
    inp = gpu_inputs(w, seed=3, grid=False)
    cfg = api.config_from_workload(w)
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias)
    layer(inp.x)
    dy = torch.randn(w.T, w.d_model, device="cuda").to(torch.bfloat16)
    a = layer.backward(inp.x, dy)
    b = layer.backward(inp.x, dy)
    for k in a:
        if a[k] is not None:
            assert torch.equal(a[k], b[k]), k
