"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

* Integer / index work and the fp32 gating arithmetic are compared bit for
  bit: router logits and routing on grid inputs (exact fp32 logits), the
  gate from oracle-computed logits, the permutation from oracle routing.
* Floating-point outputs are compared with max |y - y_ref| <= tol * rms(y_ref)
  plus half an ulp of y_ref in the output format (the output's own storage
  rounding), tol = 2e-2 for bf16 and 1e-4 for fp32.
* Sizes: shape-reduced workloads (several tiles, ragged tails, partial N
  tiles) compared element by element; the full workload sizes run
  moe_forward exactly as the benchmark launches it and compare the full
  routing plus a sample of output tokens.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS, make_inputs, router_sum_bound
from oracle import moe_oracle as O
from tests.gpu_common import (SMALL, TOL, LazyExperts, assert_close_rms, gpu_inputs, half_ulp,
                              oracle_config, output_margins, record_margin, state_dev, state_np,
                              to_f64, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    api.lib()
    yield
    torch.cuda.synchronize()


def _bias_np(inp):
    return None if inp.bias is None else to_np(inp.bias)


def _route_gpu(cfg, inp):
    B = api.step_buffers(cfg)
    api.moe_route(cfg, inp.x, inp.w_router, inp.bias, B.logits, B.probs, B.topk_idx, B.topk_gate, B.ws,
                  route_state=inp.route_state)
    return B


# ---------------------------------------------------------------------------
# steps 1-3a
# ---------------------------------------------------------------------------

# extra routing cases: the fused CUDA-core router (E <= 32 and W_r within
# 200 KB of shared memory; 8, 16 and 32 accumulators a lane) and the tcgen05
# router GEMM, K whole or split
ROUTE_EXTRA = {
    # fp32, E <= 32: the logits come from the gate kernel's own CUDA-core router
    "fused_router_f32_s": replace(WORKLOADS["tiny_f32"], T=300, d_model=512),
    "fused_router_e32_f32_s": replace(WORKLOADS["tiny_f32"], T=200, E=32, d_model=256),
    # bf16, E <= 32: the same fused router on bf16 x and W_r
    "fused_router_bf16_s": replace(WORKLOADS["gshard"], T=300),
    "fused_router_e32_bf16_s": replace(WORKLOADS["gshard"], T=200, E=32, d_model=512),
    # bf16, E = 32 with a 256 KB W_r: the tcgen05 router GEMM, one K part
    "router_gemm_e32_s": replace(WORKLOADS["gshard"], T=200, E=32, d_model=4096),
    # E > 32: the tcgen05 router GEMM with K split over CTAs
    "split_k_s": replace(WORKLOADS["deepseekmoe_tc"], T=300),
    "split_k_groups_s": replace(WORKLOADS["deepseek_v2"], T=200, d_model=1024, keep_num=0, keep_den=0),
    # the router GEMM with the gate in its epilogue (clusters of 4 or 2 K
    # parts): a last 256-token tile with no second half (T = 800), two K
    # parts (K / 64 not a multiple of 4; more tiles than a wave of clusters
    # of 4), every expert count a lane is built for (E = 8 ... 256), lanes
    # past E, groups across lanes and of two a lane, the three routing
    # rules, renormalisation, expert choice
    "tc_tail_groups_s": replace(WORKLOADS["deepseek_v2"], T=800, d_model=1024, keep_num=0, keep_den=0),
    "tc_ks2_s": replace(WORKLOADS["deepseekmoe_tc"], T=300, d_model=384),
    "tc_ks2_many_tiles_s": replace(WORKLOADS["deepseekmoe_tc"], T=9700, d_model=256),
    "tc_e8_s": replace(WORKLOADS["mixtral"], T=300),
    "tc_e33_s": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=33, S=0, k=4, d_model=256),
    "tc_e96_ec_s": replace(WORKLOADS["deepseekmoe_ec"], T=320, E=96, S=0, d_model=256, ec_capacity=20),
    "tc_e128_renorm_s": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=128, S=0, k=8, d_model=256,
                                renormalize=True),
    "tc_e192_load_s": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=192, S=0, k=2, d_model=256,
                              route_rule="load", route_alpha=0.5),
    "tc_e100_groups_s": replace(WORKLOADS["deepseek_v2"], T=300, E=100, n_groups=4, topk_groups=2, k=5,
                                d_model=256, keep_num=0, keep_den=0),
    "tc_e64_groups16_s": replace(WORKLOADS["deepseek_v2"], T=300, E=64, n_groups=16, topk_groups=3, k=6,
                                 d_model=256, keep_num=0, keep_den=0),
    "tc_e224_bias_s": replace(WORKLOADS["deepseek_v3"], T=300, E=224, d_model=512),
    # one token (three of a cluster's four CTAs own no token), and a ragged
    # 32-token unit
    "tc_t1_s": replace(WORKLOADS["deepseek_v2"], T=1, d_model=256, keep_num=0, keep_den=0),
    "tc_t33_s": replace(WORKLOADS["deepseek_v2"], T=33, d_model=512, keep_num=0, keep_den=0),
}


@pytest.mark.parametrize("name", list(SMALL) + list(ROUTE_EXTRA) + ["full:" + n for n in WORKLOADS])
def test_route_bit_exact(name):
    """Router GEMM (tcgen05 for bf16, CUDA cores for fp32) + gate, grid inputs."""
    w = (WORKLOADS[name[5:]] if name.startswith("full:")
         else ROUTE_EXTRA[name] if name in ROUTE_EXTRA else SMALL[name])
    inp = make_inputs(w, seed=1, device="cuda", grid=True, with_weights=False)
    # grid inputs: every partial sum of a router dot product stays below 2^10
    # (products are multiples of 2^-13), so the fp32 logits are exact in any order
    assert router_sum_bound(inp) < 2.0 ** 10
    cfg = api.config_from_workload(w)
    B = _route_gpu(cfg, inp)
    torch.cuda.synchronize()
    ref_l = O.router_logits(to_np(inp.x), to_np(inp.w_router), _bias_np(inp))
    assert np.array_equal(to_np(B.logits), ref_l)
    probs, idx, gate, _ = O.route(oracle_config(w), ref_l, state_np(inp))
    assert np.array_equal(to_np(B.probs), probs)
    if w.mode == "tc":
        assert np.array_equal(to_np(B.topk_idx), idx)
        assert np.array_equal(to_np(B.topk_gate), gate)
    api.moe_check_device_errors(B.ws)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_gate_bit_exact_from_oracle_logits(name):
    """Softmax / top-k / group limit on normal (non-grid) inputs, full size."""
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=2, device="cpu", grid=False, with_weights=False)
    ref_l = O.router_logits(to_np(inp.x), to_np(inp.w_router), _bias_np(inp))
    probs, idx, gate, _ = O.route(oracle_config(w), ref_l, state_np(inp))
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    api.moe_gate(cfg, torch.from_numpy(ref_l).cuda(), B.probs, B.topk_idx, B.topk_gate, B.ws,
                 route_state=state_dev(inp))
    torch.cuda.synchronize()
    assert np.array_equal(to_np(B.probs), probs)
    if w.mode == "tc":
        assert np.array_equal(to_np(B.topk_idx), idx)
        assert np.array_equal(to_np(B.topk_gate), gate)


GATE_EXTRA = {
    # eight lanes a token with 12, 16 and 24 experts a lane; a lane range past E
    "e33": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=33, S=0, k=4, zipf_s=0.0),
    "e96": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=96, S=0, k=6, zipf_s=0.0),
    "e128_renorm": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=128, S=0, k=8, zipf_s=0.0,
                           renormalize=True),
    "e192_load": replace(WORKLOADS["deepseekmoe_tc"], T=300, E=192, S=0, k=2, zipf_s=0.0,
                         route_rule="load", route_alpha=0.5),
    # groups that straddle lanes (25 experts a group, 13 a lane) and groups of
    # 4 (two groups a lane)
    "e100_groups": replace(WORKLOADS["deepseek_v2"], T=300, E=100, n_groups=4, topk_groups=2, k=5,
                           keep_num=0, keep_den=0),
    "e64_groups16": replace(WORKLOADS["deepseek_v2"], T=300, E=64, n_groups=16, topk_groups=3, k=6,
                            keep_num=0, keep_den=0),
    # expert choice on the same kernel (probabilities only)
    "e96_ec": replace(WORKLOADS["deepseekmoe_ec"], T=320, E=96, S=0, zipf_s=0.0, ec_capacity=20),
}


@pytest.mark.parametrize("name", list(GATE_EXTRA))
def test_gate_bit_exact_more_experts(name):
    """Softmax / group limit / top-k for more than 32 experts (eight lanes a
    token) on the oracle's logits: every expert count per lane the kernel
    is built for, lanes past E, groups across lanes, the routing rules."""
    w = GATE_EXTRA[name]
    inp = make_inputs(w, seed=19, device="cpu", grid=False, with_weights=False)
    ref_l = O.router_logits(to_np(inp.x), to_np(inp.w_router), _bias_np(inp))
    probs, idx, gate, _ = O.route(oracle_config(w), ref_l, state_np(inp))
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    api.moe_gate(cfg, torch.from_numpy(ref_l).cuda(), B.probs, B.topk_idx, B.topk_gate, B.ws,
                 route_state=state_dev(inp))
    torch.cuda.synchronize()
    assert np.array_equal(to_np(B.probs), probs)
    if w.mode == "tc":
        assert np.array_equal(to_np(B.topk_idx), idx)
        assert np.array_equal(to_np(B.topk_gate), gate)


def test_gate_ties_go_to_the_lower_expert():
    """Logits with many exact ties (a grid of quarters): the lower expert
    index wins every tie, across the eight lanes and inside one."""
    w = replace(WORKLOADS["deepseekmoe_tc"], T=256, E=160, S=0, k=6, zipf_s=0.0)
    rng = np.random.default_rng(23)
    ref_l = (rng.integers(-4, 5, size=(w.T, w.E)) / 4.0).astype(np.float32)
    probs, idx, gate, _ = O.route(oracle_config(w), ref_l, None)
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    api.moe_gate(cfg, torch.from_numpy(ref_l).cuda(), B.probs, B.topk_idx, B.topk_gate, B.ws)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(B.probs), probs)
    assert np.array_equal(to_np(B.topk_idx), idx)
    assert np.array_equal(to_np(B.topk_gate), gate)


def _route_exact_logits(w, ref_l):
    """moe_route on x carrying `ref_l` (exact in bf16) in its first E columns
    and W_r the identity on them, so that l = x W_r^T is exactly ref_l."""
    x = torch.zeros(w.T, w.d_model, dtype=torch.float32)
    x[:, :w.E] = torch.from_numpy(ref_l)
    wr = torch.zeros(w.E, w.d_model, dtype=torch.float32)
    wr[:, :w.E] = torch.eye(w.E)
    x, wr = x.to(torch.bfloat16).cuda(), wr.to(torch.bfloat16).cuda()
    assert torch.equal(x[:, :w.E].float().cpu(), torch.from_numpy(ref_l))
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    api.moe_route(cfg, x, wr, None, B.logits, B.probs, B.topk_idx, B.topk_gate, B.ws)
    torch.cuda.synchronize()
    api.moe_check_device_errors(B.ws)
    return B


def test_fused_router_gate_quotients_below_the_normal_range():
    """Probabilities below 2^-126 (logits 82-87 below the token's maximum):
    the fused gate's division then takes the IEEE quotient instead of the
    fp64-reciprocal product; both must round exactly as the oracle's fp32
    division, subnormal results included."""
    w = replace(WORKLOADS["deepseek_v2"], T=300, d_model=256, keep_num=0, keep_den=0)
    rng = np.random.default_rng(31)
    ref_l = np.zeros((w.T, w.E), dtype=np.float32)
    far = np.float32([-82.0, -83.0, -84.5, -85.0, -86.0, -86.5, -87.0, -88.0, -90.0])
    ref_l[:] = far[rng.integers(0, len(far), size=(w.T, w.E))]
    ref_l[np.arange(w.T), rng.integers(0, w.E, size=w.T)] = 0.0      # one maximum a token
    ref_l[: w.T // 2] = np.where(rng.random((w.T // 2, w.E)) < 0.5, ref_l[: w.T // 2],
                                 (rng.integers(-8, 1, size=(w.T // 2, w.E)) / 2.0).astype(np.float32))
    probs, idx, gate, _ = O.route(oracle_config(w), ref_l, None)
    assert (probs[probs > 0] < 2.0 ** -126).any(), "some probabilities must be subnormal"
    B = _route_exact_logits(w, ref_l)
    assert np.array_equal(to_np(B.probs), probs)
    assert np.array_equal(to_np(B.topk_idx), idx)
    assert np.array_equal(to_np(B.topk_gate), gate)


@pytest.mark.parametrize("groups", [False, True])
def test_fused_router_gate_ties_go_to_the_lower_expert(groups):
    """The gate inside the router GEMM's epilogue on logits with many exact
    ties: x carries the wanted logits (quarters, exact in bf16) in its first
    E columns and W_r is the identity on them, so l = x W_r^T is exactly
    those values; moe_route must then route like the oracle, bit for bit,
    with the lower expert (and group) index winning every tie."""
    w = replace(WORKLOADS["deepseek_v2"], T=600, d_model=256, keep_num=0, keep_den=0,
                **({} if groups else {"n_groups": 0, "topk_groups": 0}))
    rng = np.random.default_rng(29)
    ref_l = (rng.integers(-4, 5, size=(w.T, w.E)) / 4.0).astype(np.float32)
    probs, idx, gate, _ = O.route(oracle_config(w), ref_l, None)
    B = _route_exact_logits(w, ref_l)
    assert np.array_equal(to_np(B.logits), ref_l)
    assert np.array_equal(to_np(B.probs), probs)
    assert np.array_equal(to_np(B.topk_idx), idx)
    assert np.array_equal(to_np(B.topk_gate), gate)


# ---------------------------------------------------------------------------
# steps 3b-4
# ---------------------------------------------------------------------------

def _permute_check(w, seed=3, bias_override=None):
    inp = make_inputs(w, seed=seed, device="cpu", grid=False, with_weights=False)
    bias = _bias_np(inp) if bias_override is None else bias_override
    ref_l = O.router_logits(to_np(inp.x), to_np(inp.w_router), bias)
    oc = oracle_config(w)
    probs, idx, gate, disp = O.route(oc, ref_l, state_np(inp))
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    xg = inp.x.cuda()
    tk_i = torch.from_numpy(idx).cuda() if idx is not None else None
    tk_g = torch.from_numpy(gate).cuda() if gate is not None else None
    api.moe_permute(cfg, xg, tk_i, tk_g, torch.from_numpy(probs).cuda(), B.counts, B.offsets,
                    B.tok_rows, B.row_token, B.row_gate, B.x_perm, B.n_dropped, B.ws)
    torch.cuda.synchronize()
    R = int(disp.offsets[-1])
    assert np.array_equal(to_np(B.counts), disp.counts)
    assert np.array_equal(to_np(B.offsets), disp.offsets)
    assert int(B.n_dropped.item()) == disp.n_dropped
    assert np.array_equal(to_np(B.tok_rows), disp.tok_rows.reshape(-1))
    assert np.array_equal(to_np(B.row_token)[:R], disp.row_token)
    assert np.array_equal(to_np(B.row_gate)[:R], disp.row_gate)
    # x_perm rows are byte copies of the x rows they name
    assert torch.equal(B.x_perm[:R], xg[B.row_token[:R].long()])
    api.moe_check_device_errors(B.ws)
    return disp


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_permute_bit_exact_full_size(name):
    _permute_check(WORKLOADS[name])


@pytest.mark.parametrize("name", list(SMALL))
def test_permute_bit_exact_small(name):
    _permute_check(SMALL[name])


def test_permute_capacity_saturated():
    """Every token's first choice is expert 0: exactly C of them survive."""
    w = SMALL["gshard_s"]
    bias = np.zeros(w.E, np.float32)
    bias[0] = 100.0
    disp = _permute_check(w, bias_override=bias)
    C = O.capacity_from_factor(w.T, w.E, w.k, w.capacity_factor)
    assert disp.kept[0] == C and disp.n_dropped > 0


def test_permute_unused_experts():
    """Half of the experts receive no token at all (empty segments)."""
    w = SMALL["dsmoe_tc_s"]
    bias = np.zeros(w.E, np.float32)
    bias[w.E // 2:] = -1.0e4
    disp = _permute_check(w, bias_override=bias)
    assert np.all(disp.counts[w.E // 2:] == 0)


# ---------------------------------------------------------------------------
# step 5
# ---------------------------------------------------------------------------

def _ffn_reference_rows(w, oc, inp_np, disp, T, lazy):
    """Oracle y_rows: gate * FFN_e(x_t) per routed row, FFN_s(x_t) per shared row."""
    x = inp_np
    R = int(disp.offsets[-1])
    rows = {}
    for e in range(w.E):
        a, b = int(disp.offsets[e]), int(disp.offsets[e + 1])
        if b > a:
            out = O.expert_ffn(x[disp.row_token[a:b]], lazy["w1"][e], lazy["w2"][e], lazy["w3"][e], w.act)
            rows[e] = out * disp.row_gate[a:b, None].astype(np.float64)
    shared = [O.expert_ffn(x, lazy["w1"][w.E + s], lazy["w2"][w.E + s], lazy["w3"][w.E + s], w.act)
              for s in range(w.S)]
    return R, rows, shared


def _assert_rows_close(y, ref, dtype, what):
    """Per row: max(|y - ref| - half an ulp of ref in the rows' storage
    format) <= TOL[dtype] * rms(row) (the rule of the layer output, P17 of
    the design notes, row by row)."""
    tol = TOL[dtype]
    rms = np.sqrt(np.mean(ref ** 2, axis=1)) + 1e-30
    err = (np.abs(y - ref) - half_ulp(ref, dtype)).max(axis=1)
    worst = int(np.argmax(err / rms))
    assert np.all(err <= tol * rms), (f"{what}: row {worst} max(|err| - half ulp) {err[worst]:.3e} > "
                                      f"{tol} * row rms {rms[worst]:.3e}")
    return float(err[worst] / rms[worst])


@pytest.mark.parametrize("grid", [True, False], ids=["grid", "normal"])
@pytest.mark.parametrize("name", list(SMALL))
def test_expert_ffn_rows(name, grid):
    """moe_expert_ffn on the oracle's routing, row by row; x either on the
    routing grid or plain N(0, 1) (the benchmark's activations)."""
    w = SMALL[name]
    inp = gpu_inputs(w, seed=4, grid=grid)
    oc = oracle_config(w)
    x_np = to_np(inp.x)
    ref_l = O.router_logits(x_np, to_np(inp.w_router), _bias_np(inp))
    probs, idx, gate, disp = O.route(oc, ref_l, state_np(inp))
    cfg = api.config_from_workload(w)
    s = api.query_sizes(cfg)
    B = api.step_buffers(cfg)
    R = int(disp.offsets[-1])
    B.offsets.copy_(torch.from_numpy(disp.offsets))
    B.row_gate[:R].copy_(torch.from_numpy(disp.row_gate))
    B.x_perm[:R].copy_(inp.x[torch.from_numpy(disp.row_token).long().cuda()])
    api.moe_expert_ffn(cfg, inp.x, B.x_perm, B.offsets, B.row_gate, inp.w1, inp.w3, inp.w2, B.h,
                       B.y_rows, B.ws)
    torch.cuda.synchronize()
    lazy = {"w1": LazyExperts(inp.w1), "w2": LazyExperts(inp.w2), "w3": LazyExperts(inp.w3)}
    R, rows, shared = _ffn_reference_rows(w, oc, x_np, disp, w.T, lazy)
    y_rows = to_f64(B.y_rows)
    ref = np.zeros((R, w.d_model))
    for e, out in rows.items():
        ref[disp.offsets[e]:disp.offsets[e + 1]] = out
    # each row is one expert's output for one token: the tolerance rule is
    # applied per row (rows differ in scale by their gates)
    worst = _assert_rows_close(y_rows[:R], ref, w.dtype, "routed rows")
    for si, sh in enumerate(shared):
        base = s.rows_cap + si * w.T
        worst = max(worst, _assert_rows_close(y_rows[base:base + w.T], sh, w.dtype, f"shared expert {si}"))
    record_margin(f"expert_rows_{'grid' if grid else 'normal'}:{w.name}:T={w.T}",
                  {"worst_row_excess_over_rms": worst, "tol": TOL[w.dtype]})
    api.moe_check_device_errors(B.ws)


@pytest.mark.parametrize("name", list(SMALL))
def test_combine_sums_rows_in_order(name):
    w = SMALL[name]
    inp = make_inputs(w, seed=5, device="cpu", grid=False, with_weights=False)
    oc = oracle_config(w)
    ref_l = O.router_logits(to_np(inp.x), to_np(inp.w_router), _bias_np(inp))
    _, _, _, disp = O.route(oc, ref_l, state_np(inp))
    cfg = api.config_from_workload(w)
    s = api.query_sizes(cfg)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    y_rows = torch.randn(s.rows_total, w.d_model, generator=g, device="cuda").to(dt)  # layer dtype
    tok_rows = torch.from_numpy(disp.tok_rows.reshape(-1).copy()).cuda()
    y = torch.empty(w.T, w.d_model, dtype=dt, device="cuda")
    api.moe_combine(cfg, y_rows, tok_rows, y)
    torch.cuda.synchronize()
    yr = to_f64(y_rows)
    ref = np.zeros((w.T, w.d_model))
    for t in range(w.T):
        rows = (disp.tok_rows[:, t] if w.mode == "ec" else disp.tok_rows[t])
        for r in rows:
            if r >= 0:
                ref[t] += yr[r]
        for si in range(w.S):
            ref[t] += yr[s.rows_cap + si * w.T + t]
    got = to_f64(y)
    # fp32 accumulation then one rounding to the output type
    ulp = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -23
    bound = ulp * np.abs(ref) + 1e-5 * (1 + np.abs(yr).max())
    assert np.all(np.abs(got - ref) <= bound)


# ---------------------------------------------------------------------------
# steps 1-5 through moe_forward
# ---------------------------------------------------------------------------

def _forward_check(w, seed=6, tokens=None, inp=None):
    inp = inp if inp is not None else gpu_inputs(w, seed=seed, grid=True)
    cfg = api.config_from_workload(w)
    ws = api.new_workspace(cfg)
    y = torch.empty_like(inp.x)
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, counts, ws,
                    route_state=inp.route_state)
    api.moe_check_device_errors(ws)
    oc = oracle_config(w)
    x_np = to_np(inp.x)
    ref_l = O.router_logits(x_np, to_np(inp.w_router), _bias_np(inp))
    probs, idx, gate, disp = O.route(oc, ref_l, state_np(inp))
    assert np.array_equal(to_np(counts), disp.counts)
    toks = np.arange(w.T) if tokens is None else np.asarray(tokens)
    lazy = (LazyExperts(inp.w1), LazyExperts(inp.w2), LazyExperts(inp.w3))
    ref = O.combine_tokens(oc, x_np, lazy[0], lazy[1], lazy[2], disp, toks)
    got = to_f64(y)[toks]
    rel = assert_close_rms(got, ref, w.dtype)
    record_margin(f"forward_grid:{w.name}:T={w.T}", output_margins(got, ref, w.dtype))
    return rel, disp


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small(name):
    _forward_check(SMALL[name])


FOLDED = [n for n, w in SMALL.items()
          if w.dtype == "bf16" and w.mode == "tc" and w.k + w.S <= 2]


@pytest.mark.parametrize("name", FOLDED + ["full:gshard", "full:mixtral"])
def test_folded_combine_equals_the_steps(name):
    """With at most two rows a token, moe_forward adds the gated rows into y
    inside the down-projection; the result is bit-identical to the step entry
    points (gated rows written out, then the combine kernel's fp32 sum and one
    rounding)."""
    w = WORKLOADS[name[5:]] if name.startswith("full:") else SMALL[name]
    inp = gpu_inputs(w, seed=12, grid=False)
    cfg = api.config_from_workload(w)
    ws = api.new_workspace(cfg)
    y = torch.empty_like(inp.x)
    api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, None, ws,
                    route_state=inp.route_state)
    B = api.step_buffers(cfg)
    api.moe_route(cfg, inp.x, inp.w_router, inp.bias, B.logits, B.probs, B.topk_idx, B.topk_gate,
                  B.ws, route_state=inp.route_state)
    api.moe_permute(cfg, inp.x, B.topk_idx, B.topk_gate, B.probs, B.counts, B.offsets, B.tok_rows,
                    B.row_token, B.row_gate, B.x_perm, B.n_dropped, B.ws)
    api.moe_expert_ffn(cfg, inp.x, B.x_perm, B.offsets, B.row_gate, inp.w1, inp.w3, inp.w2, B.h,
                       B.y_rows, B.ws)
    y_steps = torch.empty_like(inp.x)
    api.moe_combine(cfg, B.y_rows, B.tok_rows, y_steps)
    torch.cuda.synchronize()
    api.moe_check_device_errors(ws)
    api.moe_check_device_errors(B.ws)
    assert torch.equal(y.view(torch.int16), y_steps.view(torch.int16))


def _steps_from_oracle_logits(w, seed=13, tokens=None):
    """The whole layer through the step entry points on plain N(0, 1) inputs
    (no grid): the oracle's fp32 router logits go to moe_gate (so routing is
    defined by identical logits, and checked bit for bit), then moe_permute,
    moe_expert_ffn and moe_combine; y is compared with the oracle's
    float64 forward element by element (P17, with its margin recorded), and
    with the oracle's output rounded once to the output format."""
    inp = gpu_inputs(w, seed=seed, grid=False)
    oc = oracle_config(w)
    x_np = to_np(inp.x)
    ref_l = O.router_logits(x_np, to_np(inp.w_router), _bias_np(inp))
    probs, idx, gate, disp = O.route(oc, ref_l, state_np(inp))
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    api.moe_gate(cfg, torch.from_numpy(ref_l).cuda(), B.probs, B.topk_idx, B.topk_gate, B.ws,
                 route_state=state_dev(inp))
    api.moe_permute(cfg, inp.x, B.topk_idx, B.topk_gate, B.probs, B.counts, B.offsets, B.tok_rows,
                    B.row_token, B.row_gate, B.x_perm, B.n_dropped, B.ws)
    api.moe_expert_ffn(cfg, inp.x, B.x_perm, B.offsets, B.row_gate, inp.w1, inp.w3, inp.w2, B.h,
                       B.y_rows, B.ws)
    api.moe_combine(cfg, B.y_rows, B.tok_rows, B.y)
    torch.cuda.synchronize()
    api.moe_check_device_errors(B.ws)
    if w.mode == "tc":
        assert np.array_equal(to_np(B.topk_idx), idx)
    assert np.array_equal(to_np(B.offsets), disp.offsets)
    assert np.array_equal(to_np(B.tok_rows), disp.tok_rows.reshape(-1))
    toks = np.arange(w.T) if tokens is None else np.asarray(tokens)
    lazy = (LazyExperts(inp.w1), LazyExperts(inp.w2), LazyExperts(inp.w3))
    ref = O.combine_tokens(oc, x_np, lazy[0], lazy[1], lazy[2], disp, toks)
    got = to_f64(B.y)[toks]
    m = output_margins(got, ref, w.dtype)
    record_margin(f"steps_normal:{w.name}:T={w.T}", m)
    assert m["excess_over_rms"] <= TOL[w.dtype], m
    assert m["vs_rounded_ref_over_rms"] <= TOL[w.dtype], m
    return m


@pytest.mark.parametrize("name", list(SMALL))
def test_steps_normal_inputs_small(name):
    _steps_from_oracle_logits(SMALL[name])


@pytest.mark.parametrize("name", ["gshard", "mixtral", "deepseekmoe_tc", "deepseekmoe_ec",
                                  "deepseek_v2"])
def test_steps_normal_inputs_full_size_sampled(name):
    """Full workload sizes, plain N(0, 1) activations, 24 sampled tokens."""
    w = WORKLOADS[name]
    rng = np.random.default_rng(17)
    toks = np.unique(np.concatenate([[0, w.T - 1], rng.integers(0, w.T, 22)]))
    _steps_from_oracle_logits(w, tokens=toks)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_forward_full_size_sampled(name):
    """The benchmark's launch configuration at full size: full routing bit-exact
    (counts), outputs of 24 sampled tokens (first, last, 22 seeded) within tolerance."""
    w = WORKLOADS[name]
    rng = np.random.default_rng(11)
    toks = np.unique(np.concatenate([[0, w.T - 1], rng.integers(0, w.T, 22)]))
    _forward_check(w, seed=6, tokens=toks)
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 2, 127, 129])
@pytest.mark.parametrize("base", ["gshard_s", "dsmoe_ec_s", "dsv2_s", "tiny_f32"])
def test_forward_ragged_token_counts(T, base):
    _forward_check(SMALL[base].with_tokens(T))


def test_dense_mixture_k_equals_E():
    w = replace(SMALL["mixtral_s"], T=200, k=8, renormalize=False)
    _forward_check(w)


def test_single_expert_dense_ffn():
    w = replace(SMALL["gshard_s"], T=300, E=1, k=1, capacity_factor=0.0)
    _forward_check(w)


@pytest.mark.parametrize("base,S", [("dsv3_s", 8), ("dsmoe_tc_s", 8), ("tiny_f32", 3)])
def test_forward_most_shared_experts(base, S):
    """The largest shared-expert count the library takes (8): with the V3
    shape's 256 routed experts that is 264 weight groups in one grouped GEMM;
    and shared experts on the fp32 path."""
    _forward_check(replace(SMALL[base], S=S, T=300))


def test_all_routed_dropped_leaves_shared_experts():
    w = replace(SMALL["dsv2_s"], T=300, keep_num=0, keep_den=1)
    rel, disp = _forward_check(w)
    assert disp.n_dropped == w.T * w.k


@pytest.mark.parametrize("T", [255, 256, 257, 512, 513, 1000])
def test_token_tiles_of_one_hot_expert(T):
    """Short experts run on token-N tiles (weights on the MMA's M side, up to
    256 tokens a tile, widths cut to multiples of 32): a strong Zipf bias
    sends nearly every token to expert 0, whose segment of about T rows is cut
    into ceil(T / 256) tiles, the others staying short or empty."""
    w = replace(SMALL["gshard_s"], T=T, E=4, k=1, capacity_factor=0.0, zipf_s=12.0)
    rel, disp = _forward_check(w)
    assert disp.counts[0] >= T - 8


@pytest.mark.parametrize("name", ["dsv2_s", "mixtral_s", "fold_shared_s"])
def test_token_n_expert_gemms_match_the_tile_kernel(name):
    """The token-N expert GEMMs give, within rounding, what the 128-row tile
    kernel gives: both paths compared with the oracle on the same inputs is
    the real check (test_forward_small); here the layer output of the token-N
    path is also checked on plain N(0, 1) activations at the workload's
    shape, through the step entry points."""
    _steps_from_oracle_logits(SMALL[name], seed=41)


def test_expert_choice_takes_every_token():
    w = replace(SMALL["dsmoe_ec_s"], T=200, ec_capacity=200)
    _forward_check(w)


def test_bad_expert_index_sets_the_error_word():
    """A corrupted routing index is caught by the kernel's own check: the
    error word reports it and nothing out of range is touched."""
    w = SMALL["gshard_s"]
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    x = torch.randn(w.T, w.d_model, device="cuda").to(torch.bfloat16)
    idx = torch.randint(0, w.E, (w.T, w.k), device="cuda", dtype=torch.int32)
    idx[:, 1] = (idx[:, 0] + 1) % w.E
    idx[5, 0] = w.E + 3
    gate = torch.rand(w.T, w.k, device="cuda")
    api.moe_permute(cfg, x, idx, gate, None, B.counts, B.offsets, B.tok_rows, B.row_token,
                    B.row_gate, B.x_perm, B.n_dropped, B.ws)
    with pytest.raises(api.MoeError) as ei:
        api.moe_check_device_errors(B.ws)
    assert ei.value.status == api.MOE_ERR_DEVICE_CHECK
    # the word is cleared after reading
    assert api.moe_check_device_errors(B.ws) == 0
