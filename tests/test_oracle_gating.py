"""Pins of the oracle's gating steps (router logits, softmax, exp).

Each check ties the oracle to something other than itself: float64
mathematics (math.exp, torch float64 softmax), hand-worked values under
tests/golden/, or properties that hold for any correct softmax.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _ulp_err(got: np.ndarray, z: np.ndarray) -> np.ndarray:
    """Distance in fp32 ulps between got and the float64 exp(z)."""
    ref = np.exp(z.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    return np.abs(got.astype(np.float64) - ref) / ulp


def test_exp_det_within_two_ulp():
    rng = np.random.default_rng(0)
    z = np.concatenate([
        np.linspace(-87.0, 0.0, 400001, dtype=np.float32),
        rng.uniform(-87.0, 0.0, 400000).astype(np.float32),
        -np.logspace(-12, 0, 20000).astype(np.float32),
        (np.arange(-125, 1) * np.float32(math.log(2.0))).astype(np.float32),
    ])
    got = O.exp_det(z)
    err = _ulp_err(got, z)
    assert err.max() <= 2.0, f"max ulp error {err.max()}"


def test_exp_det_special_values():
    assert O.exp_det(np.array([0.0], np.float32))[0] == np.float32(1.0)
    assert O.exp_det(np.array([-0.0], np.float32))[0] == np.float32(1.0)
    # below the flush threshold the result is exactly zero
    z = np.array([-87.5, -100.0, -1e30], np.float32)
    assert np.all(O.exp_det(z) == 0.0)
    # just above it: a normal positive number near exp(-87)
    v = O.exp_det(np.array([-87.0], np.float32))[0]
    assert v > 0 and abs(v / math.exp(-87.0) - 1.0) < 1e-6


def test_softmax_matches_float64_closed_form():
    rng = np.random.default_rng(1)
    for E in (1, 2, 8, 16, 64, 160, 256):
        l = (rng.standard_normal((257, E)) * 3.0).astype(np.float32)
        p = O.softmax_det(l)
        ref = torch.softmax(torch.from_numpy(l.astype(np.float64)), dim=1).numpy()
        # bound: rounding z = l - m moves exp(z) by up to |z| * 2**-24 relative;
        # exp_det adds <= 2 ulp, the sequential fp32 sum <= E-1 roundings and
        # the division one more
        z = np.abs(l.astype(np.float64) - l.max(1, keepdims=True))
        tol = (z + 4.0 + E) * 2.0 ** -24 * ref + 1e-30
        assert np.all(np.abs(p - ref) <= tol), E
        s = p.astype(np.float64).sum(axis=1)
        assert np.all(np.abs(s - 1.0) <= (E + 4) * 2.0 ** -23)


def test_softmax_golden():
    g = json.load(open(os.path.join(GOLD, "gating_worked.json")))
    for case in g["softmax_cases"]:
        l = np.array(case["logits"], np.float32)
        p = O.softmax_det(l)
        assert np.array_equal(p, np.array(case["probs"], np.float32)), case["why"]


def test_softmax_monotone_in_logit():
    # softmax preserves the order of the logits within a token
    rng = np.random.default_rng(2)
    l = (rng.standard_normal((100, 32)) * 2).astype(np.float32)
    p = O.softmax_det(l)
    for t in range(100):
        o = np.argsort(l[t])
        assert np.all(np.diff(p[t][o]) >= 0)


def test_router_logits_float64_dot():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((33, 96)).astype(np.float32)
    w = (rng.standard_normal((12, 96)) * 0.1).astype(np.float32)
    b = rng.standard_normal(12).astype(np.float32)
    got = O.router_logits(x, w, b)
    ref = torch.nn.functional.linear(torch.from_numpy(x).double(), torch.from_numpy(w).double(),
                                     torch.from_numpy(b).double()).numpy().astype(np.float32)
    assert np.array_equal(got, ref)
    # the bias enters as a per-expert shift
    nob = O.router_logits(x, w, None)
    assert np.allclose(got.astype(np.float64) - nob, b[None, :], atol=1e-5)


def test_widen_bf16_bits():
    t = torch.tensor([1.0, -2.5, 0.0078125, 3.140625], dtype=torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.widen(bits), t.double().numpy())
