"""Planted mistakes in the oracle must trip at least one pin.

Each case patches one plausible error into the oracle (on the CPU only) and
re-runs the pin that is meant to catch it; the pin must fail.  This checks
that the pins constrain the oracle rather than restate it.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from tests import test_oracle_dispatch as TD
from tests import test_oracle_ffn as TF
from tests import test_oracle_gating as TG
from tests import test_oracle_selection as TS
from tests import test_oracle_routing_variants as TV
from tests import test_oracle_backward as TB


def _expect_pin_failure(pin, *args):
    with pytest.raises(AssertionError):
        pin(*args)


def test_token_major_priority_is_caught(monkeypatch):
    """Priority q = t*k + j (token-major) instead of j*T + t."""
    orig = O._priority_ranks

    def wrong(topk_idx, E, local_groups=1):
        T, k = topk_idx.shape
        e_tok_major = np.asarray(topk_idx, np.int64).reshape(-1)          # q' = t*k + j
        by = np.argsort(e_tok_major, kind="stable")
        # map back to the j*T + t numbering the rest of the oracle uses
        q_of_qp = (np.arange(T * k) % k) * T + np.arange(T * k) // k
        e_of_q, _, counts, start, _, g_of_q = orig(topk_idx, E, local_groups)
        rank = np.empty(T * k, np.int64)
        rank[q_of_qp[by]] = np.arange(T * k) - start[e_tok_major[by]]
        by_expert = q_of_qp[by]
        return e_of_q, by_expert, counts, start, rank, g_of_q

    monkeypatch.setattr(O, "_priority_ranks", wrong)
    _expect_pin_failure(TD.test_capacity_golden)


def test_reversed_tie_rule_is_caught(monkeypatch):
    orig = O.topk_route

    def wrong(logits, probs, k, n_groups=0, topk_groups=0, renormalize=False, rule="softmax",
              state=None, alpha=0.0):
        l = np.asarray(logits, np.float32)
        E = l.shape[1]
        st = None if state is None else np.asarray(state)[::-1]
        idx, gate = orig(l[:, ::-1], np.asarray(probs)[:, ::-1], k, n_groups, topk_groups, renormalize,
                         rule, st, alpha)
        return (E - 1 - idx).astype(np.int32), gate                    # higher index wins ties

    monkeypatch.setattr(O, "topk_route", wrong)
    _expect_pin_failure(TS.test_topk_golden)


def test_dropped_gate_is_caught(monkeypatch):
    orig = O.dispatch_token_choice

    def wrong(topk_idx, topk_gate, probs, E, capacity=0, keep_num=0, keep_den=0, local_groups=1):
        return orig(topk_idx, np.ones_like(topk_gate), probs, E, capacity, keep_num, keep_den,
                    local_groups)

    monkeypatch.setattr(O, "dispatch_token_choice", wrong)
    _expect_pin_failure(TF.test_k_equals_E_is_dense_soft_mixture, "relu")


@pytest.mark.parametrize("act", ["relu", "swiglu"])
def test_wrong_activation_is_caught(monkeypatch, act):
    orig = O.expert_ffn

    def wrong(xrows, w1_e, w2_e, w3_e=None, act="relu"):
        if act == "relu":                       # activation dropped
            return O.widen(xrows) @ O.widen(w1_e).T @ O.widen(w2_e).T
        return orig(xrows, w3_e, w2_e, w1_e, act)   # gate and up swapped

    monkeypatch.setattr(O, "expert_ffn", wrong)
    _expect_pin_failure(TF.test_single_expert_is_dense_ffn, act)


def test_missing_shared_term_is_caught(monkeypatch):
    orig = O.combine_tokens

    def wrong(cfg, x, w1, w2, w3, disp, tokens):
        cfg2 = O.OracleConfig(**{**cfg.__dict__, "S": 0})
        return orig(cfg2, x, w1, w2, w3, disp, tokens)

    monkeypatch.setattr(O, "combine_tokens", wrong)
    _expect_pin_failure(TF.test_shared_experts_alone)


def test_expert_choice_high_token_ties_is_caught(monkeypatch):
    orig = O.dispatch_expert_choice

    def wrong(probs, C):
        p = np.asarray(probs)[::-1]
        d = orig(p, C)
        T = p.shape[0]
        d.row_token = (T - 1 - d.row_token).astype(np.int32)
        return d

    monkeypatch.setattr(O, "dispatch_expert_choice", wrong)
    _expect_pin_failure(TD.test_expert_choice_golden)


def test_missing_low_ln2_correction_is_caught(monkeypatch):
    monkeypatch.setattr(O, "LN2_LO", np.float32(0.0))
    _expect_pin_failure(TG.test_exp_det_within_two_ulp)


def test_softmax_without_denominator_order_is_caught(monkeypatch):
    """Normalising by the max instead of the sum."""
    def wrong(logits):
        l = np.asarray(logits, np.float32)
        e = O.exp_det((l - l.max(1, keepdims=True)).astype(np.float32))
        return e

    monkeypatch.setattr(O, "softmax_det", wrong)
    _expect_pin_failure(TG.test_softmax_golden)


def test_keep_fraction_floor_is_caught(monkeypatch):
    monkeypatch.setattr(O, "keep_count", lambda n, a, b: (np.asarray(n) * a) // b if b > 0 else np.asarray(n))
    _expect_pin_failure(TD.test_keep_fraction_golden)


def test_group_score_sum_is_caught(monkeypatch):
    """Group score = sum of the group's logits instead of its maximum."""
    def wrong(logits, n_groups, topk_groups):
        l = np.asarray(logits, np.float32)
        T, E = l.shape
        gsz = E // n_groups
        score = l.reshape(T, n_groups, gsz).sum(axis=2)
        order = np.argsort(-score, axis=1, kind="stable")
        chosen = np.zeros((T, n_groups), bool)
        np.put_along_axis(chosen, order[:, :topk_groups], True, axis=1)
        return np.repeat(chosen, gsz, axis=1)

    monkeypatch.setattr(O, "group_limited_mask", wrong)
    _expect_pin_failure(TS.test_group_limited_brute_force)


def test_bias_rule_on_logits_is_caught(monkeypatch):
    """DeepSeek-V3 keys formed from the logits instead of the affinity p."""
    orig = O.selection_keys

    def wrong(logits, probs, rule="softmax", state=None, alpha=0.0):
        if rule == "bias":
            key = (np.asarray(logits, np.float32) + np.asarray(state, np.float32)[None, :]).astype(np.float32)
            return key, key
        return orig(logits, probs, rule, state, alpha)

    monkeypatch.setattr(O, "selection_keys", wrong)
    _expect_pin_failure(TV.test_bias_rule_brute_force, 0)


def test_load_rule_without_complement_is_caught(monkeypatch):
    """alpha * u instead of alpha * (1 - u)."""
    orig = O.selection_keys

    def wrong(logits, probs, rule="softmax", state=None, alpha=0.0):
        if rule == "load":
            off = (np.float32(alpha) * np.asarray(state, np.float32)).astype(np.float32)
            return (np.asarray(logits, np.float32) + off[None, :]).astype(np.float32), np.asarray(probs, np.float32)
        return orig(logits, probs, rule, state, alpha)

    monkeypatch.setattr(O, "selection_keys", wrong)
    _expect_pin_failure(TV.test_load_rule_brute_force, 0)


def test_bias_update_sign_is_caught(monkeypatch):
    orig = O.bias_update
    monkeypatch.setattr(O, "bias_update", lambda c, b, T, k, g: orig(c, b, T, k, -g))
    _expect_pin_failure(TV.test_bias_routing_golden)


def test_global_ranks_under_local_groups_are_caught(monkeypatch):
    """Capacity ranks counted over the whole batch instead of per group."""
    orig = O._priority_ranks

    def wrong(topk_idx, E, local_groups=1):
        e_of_q, by_expert, counts, start, rank, g_of_q = orig(topk_idx, E, 1)
        return e_of_q, by_expert, counts, start, rank, g_of_q

    monkeypatch.setattr(O, "_priority_ranks", wrong)
    _expect_pin_failure(TV.test_local_groups_are_independent_batches, 4)


def test_backward_silu_derivative_is_caught(monkeypatch):
    """SiLU'(a) taken as sigmoid(a) (the a * s * (1 - s) term dropped)."""
    def wrong(xr, a, u, h, dyr, w1_e, w2_e, w3_e, act):
        w2 = O.widen(w2_e)
        dw2 = dyr.T @ h
        dh = dyr @ w2
        if act == "relu":
            da = dh * (a > 0)
            return da @ O.widen(w1_e), da.T @ xr, None, dw2
        s = 1.0 / (1.0 + np.exp(-a))
        da = dh * u * s
        du = dh * a * s
        return da @ O.widen(w1_e) + du @ O.widen(w3_e), da.T @ xr, du.T @ xr, dw2

    monkeypatch.setattr(O, "_ffn_backward", wrong)
    _expect_pin_failure(TB.test_backward_matches_finite_differences, "renorm_swiglu_shared")


def test_backward_without_softmax_jacobian_is_caught(monkeypatch):
    """dlogits = dp (the softmax Jacobian left out)."""
    monkeypatch.setattr(O, "softmax_backward", lambda p, dp: dp)
    _expect_pin_failure(TB.test_backward_matches_finite_differences, "capacity_relu")
