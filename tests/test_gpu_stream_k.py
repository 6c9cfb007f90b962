"""The expert GEMMs' stream-K tail (tiles cut into k-block pieces spread over
all CTAs, summed by the CTA holding each tile's first k-block).

* Long contractions on few tiles: every tile of the CTA-pair kernel is cut
  into several pieces, so each finalizer adds three or more partial tiles
  (ReLU and SwiGLU up-projections, gate-scaled down-projection); the same
  contractions on the token-N tiles of short experts, which have no tail.
  (The single-CTA kernel's tail runs in the backward pass, covered by its
  tests.)
* The sum order is fixed by the tile count and the grid: two calls give the
  same bits.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS
from tests.gpu_common import SMALL, gpu_inputs
from tests.test_gpu_parity import _forward_check

pytestmark = pytest.mark.gpu

LONG_K = {
    # short experts: token-N tiles (no stream-K tail), down-projection K = 2048
    # on 3 tiles and K = 1536 with SwiGLU and shared experts
    "token_n_relu": replace(SMALL["gshard_s"], T=300, E=1, k=1, capacity_factor=0.0, d_ff=2048),
    "token_n_swiglu": replace(SMALL["dsv2_s"], T=260, d_ff=1536),
    # CTA pairs (256-row tiles): about 1050 rows per expert, K = 2048
    "pair_relu": replace(SMALL["pair_relu_s"], d_ff=2048),
    # CTA pairs, SwiGLU and shared experts, K = 1024 on the down-projection
    "pair_swiglu": replace(SMALL["pair_swiglu_s"], d_ff=1024),
    # CTA pairs, short last M-tiles cut into pieces, K = 2048
    "pair_half": replace(SMALL["pair_half_s"], d_ff=2048),
}


@pytest.mark.parametrize("name", list(LONG_K))
def test_long_contraction_split_over_ctas(name):
    _forward_check(LONG_K[name], seed=8)


@pytest.mark.parametrize("name", ["gshard", "pair_relu_s", "dsv2_s"])
def test_forward_is_deterministic(name):
    w = WORKLOADS[name] if name in WORKLOADS else SMALL[name]
    inp = gpu_inputs(w, seed=9, grid=False)
    cfg = api.config_from_workload(w)
    ws = api.new_workspace(cfg)
    ys = []
    for _ in range(2):
        y = torch.empty_like(inp.x)
        api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, None, ws)
        ys.append(y)
    api.moe_check_device_errors(ws)
    a = ys[0].view(torch.int16).cpu().numpy()
    b = ys[1].view(torch.int16).cpu().numpy()
    assert np.array_equal(a, b)
    # the flags of the tail are back at zero after every launch
    ctrl = ws[:4096].view(torch.int32).cpu().numpy()
    assert not ctrl[64:].any()
