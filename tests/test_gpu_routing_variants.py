"""Routing variants on the GPU against the oracle: DeepSeek-V3 bias routing
and its bias update, load-aware top-k, GShard local groups (bit-exact for
the integer work, the gates and the bias; outputs within the tolerance).
Shapes and full-size workloads of these variants also run in the parity
tests through SMALL / WORKLOADS."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from oracle import moe_oracle as O
from tests.gpu_common import SMALL, oracle_config, to_np
from tests.test_gpu_parity import _forward_check, _permute_check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("E,T,k", [(16, 4096, 2), (256, 8192, 8), (7, 100, 3)])
def test_bias_update_matches_oracle(E, T, k):
    rng = np.random.default_rng(E)
    counts = rng.multinomial(T * k, np.ones(E) / E).astype(np.int32)
    if T * k % E == 0:
        counts[0] = T * k // E                      # one expert exactly at the mean

    bias = (rng.standard_normal(E) * 0.01).astype(np.float32)
    c = api.MoeConfig()
    c.T, c.d_model, c.E, c.S, c.k, c.d_ff = T, 64, E, 0, k, 64
    c.dtype, c.act, c.mode = api.MOE_BF16, api.MOE_ACT_RELU, api.MOE_TOKEN_CHOICE
    c.route_rule = api.MOE_ROUTE_BIAS
    b_dev = torch.from_numpy(bias).cuda()
    api.moe_route_bias_update(c, torch.from_numpy(counts).cuda(), b_dev, 0.001)
    torch.cuda.synchronize()
    want = O.bias_update(counts, bias, T, k, 0.001)
    assert np.array_equal(b_dev.cpu().numpy(), want)


def test_bias_routing_over_training_steps():
    """Forward, then the bias step, several times: the GPU's counts and bias
    follow the oracle's (routing from the oracle's bias each step)."""
    w = SMALL["dsv3_s"]
    from tests.gpu_common import gpu_inputs
    inp = gpu_inputs(w, seed=12, grid=True)
    cfg = api.config_from_workload(w)
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias,
                         route_state=inp.route_state.clone())
    oc = oracle_config(w)
    ref_l = O.router_logits(to_np(inp.x), to_np(inp.w_router), None)
    b = inp.route_state.cpu().numpy()
    for step in range(4):
        layer(inp.x)
        layer.update_route_bias(0.002)
        torch.cuda.synchronize()
        _, _, _, disp = O.route(oc, ref_l, b)
        assert np.array_equal(layer.counts.cpu().numpy(), disp.counts), step
        b = O.bias_update(disp.counts, b, w.T, w.k, 0.002)
        assert np.array_equal(layer.route_state.cpu().numpy(), b), step
    api.moe_check_device_errors(layer.ws)


@pytest.mark.parametrize("G", [1, 2, 3, 6, 18])
def test_local_groups_permutation(G):
    """576 tokens in G groups of 576/G (a multiple of 32); capacity per group."""
    w = replace(SMALL["local_groups_s"], T=576, local_groups=G)
    _permute_check(w)


@pytest.mark.parametrize("G", [2, 6])
def test_local_groups_forward(G):
    _forward_check(replace(SMALL["local_groups_s"], T=576, local_groups=G, capacity_factor=1.0))


@pytest.mark.parametrize("alpha", [0.0, 0.5, 4.0])
def test_load_aware_forward(alpha):
    _forward_check(replace(SMALL["load_aware_s"], route_alpha=alpha))
