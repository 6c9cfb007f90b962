"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every device-side wait of the expert GEMMs is bounded; when one runs out the
kernel sets the timeout bit of the workspace's error word, drains its own
copies and tensor-core work, frees its TMEM and returns, so the context stays
usable.  Here a wait is made to run out on purpose: the stream-K finalizer
of a split tile waits for the ready flag of each later piece to reach its
count (one add per epilogue thread of the writer), and the flags are biased
far below zero beforehand, so no number of adds brings them there.  With the
wait limit set to 1 ms the forward must end quickly, moe_check_device_errors
must report MOE_ERR_TIMEOUT (and clear the control block), and a following
forward on the same workspace must match the oracle.  Nothing here traps,
faults or waits without a bound.
"""
import time
from dataclasses import replace

import numpy as np
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from oracle import moe_oracle as O
from tests.gpu_common import (SMALL, LazyExperts, assert_close_rms, gpu_inputs, oracle_config,
                              state_np, to_f64, to_np)

pytestmark = pytest.mark.gpu

SK_FLAGS_OFFSET, SK_SLOTS = 256, 192      # the stream-K ready flags in the control block

# Long contractions on few tiles: every tile is cut into pieces over the
# CTAs, so finalizers wait on other CTAs' flags.  CTA pairs: the forward's
# down-projection (about 1050 rows an expert, K = 2048).  Single CTAs: the
# backward's pre-activation and dA GEMMs (300 rows, K = d_model = 2048); the
# forward's short experts run on token-N tiles, which have no stream-K tail.
CASES = {
    "cta_pair_forward": (replace(SMALL["pair_relu_s"], d_ff=2048), False),
    "one_cta_backward": (replace(SMALL["gshard_s"], T=300, E=1, k=1, capacity_factor=0.0,
                                 d_model=2048, d_ff=256), True),
}


def _forward(cfg, inp, ws):
    y = torch.empty_like(inp.x)
    api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, None, ws,
                    route_state=inp.route_state)
    return y


@pytest.mark.parametrize("name", list(CASES))
def test_wait_that_runs_out_reports_timeout_and_leaves_the_context_usable(name):
    w, backward = CASES[name]
    inp = gpu_inputs(w, seed=31, grid=True)
    cfg = api.config_from_workload(w)
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias,
                         route_state=inp.route_state)
    ws = layer.ws
    dy = torch.randn(w.T, w.d_model, device="cuda").to(torch.bfloat16)
    _forward(cfg, inp, ws)                        # a normal pass first: no error
    if backward:
        layer.backward(inp.x, dy)
    assert api.moe_check_device_errors(ws) == 0

    if backward:
        _forward(cfg, inp, ws)
    api.moe_workspace_set_wait_limit(ws, 1_000_000)                  # 1 ms
    flags = ws[SK_FLAGS_OFFSET:SK_FLAGS_OFFSET + 4 * SK_SLOTS].view(torch.int32)
    flags.fill_(-(1 << 30))                       # never reaches the finalizers' count
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    if backward:
        layer.backward(inp.x, dy)
    else:
        _forward(cfg, inp, ws)
    with pytest.raises(api.MoeError) as ei:
        api.moe_check_device_errors(ws)           # synchronises, reads, clears the control block
    elapsed = time.perf_counter() - t0
    assert ei.value.status == api.MOE_ERR_TIMEOUT
    assert elapsed < 1.0, f"the 1 ms limit was not applied ({elapsed:.2f} s)"
    ctrl = ws[:4096].view(torch.int32).cpu().numpy()
    assert not ctrl.any(), "control block (error word, wait limit, flags) cleared after the error"

    # the same workspace, default limit: a normal forward, checked against the oracle
    y = _forward(cfg, inp, ws)
    assert api.moe_check_device_errors(ws) == 0
    oc = oracle_config(w)
    x_np = to_np(inp.x)
    bias = None if inp.bias is None else to_np(inp.bias)
    ref_l = O.router_logits(x_np, to_np(inp.w_router), bias)
    _, _, _, disp = O.route(oc, ref_l, state_np(inp))
    lazy = (LazyExperts(inp.w1), LazyExperts(inp.w2), LazyExperts(inp.w3))
    ref = O.combine_tokens(oc, x_np, lazy[0], lazy[1], lazy[2], disp, np.arange(w.T))
    assert_close_rms(to_f64(y), ref, w.dtype)


def test_wait_limit_entry_point_validates_its_workspace():
    small = torch.zeros(1024, dtype=torch.uint8, device="cuda")      # below the 4 KiB control block
    with pytest.raises(api.MoeError) as ei:
        api.moe_workspace_set_wait_limit(small, 1000)
    assert ei.value.status == api.MOE_ERR_INVALID_ARG
