"""Kernel launches of one moe_forward, counted by the library's own launch
counter (moe_kernel_launches): the structure bench.py reports as
gpu_launches.  With few experts the router runs inside the gate kernel; a
small unit histogram is summed inside the rank kernel; with at most two
rows a token the combine is folded into the down-projection."""
from dataclasses import replace

import pytest
import torch

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS
from tests.gpu_common import SMALL, gpu_inputs

pytestmark = pytest.mark.gpu

CASES = {
    # router+gate, rank (own unit sums), gather, up, down (combine folded)
    "gshard": (WORKLOADS["gshard"], 5),
    "gshard_s": (SMALL["gshard_s"], 5),
    # d = 4096: the tcgen05 router GEMM with the gate in its epilogue
    "mixtral": (WORKLOADS["mixtral"], 5),
    # E = 64, k = 6 with shared experts: router GEMM + gate, rank, gather, up, down, combine;
    # the 3072-unit histogram is summed by its own kernel
    "deepseekmoe_tc": (WORKLOADS["deepseekmoe_tc"], 7),
    # a small histogram with k + S > 2: the combine runs
    "dsmoe_tc_s": (SMALL["dsmoe_tc_s"], 6),
}


@pytest.mark.parametrize("name", list(CASES))
def test_kernels_per_forward(name):
    w, expected = CASES[name]
    inp = gpu_inputs(w, seed=13, grid=False)
    cfg = api.config_from_workload(w)
    ws = api.new_workspace(cfg)
    y = torch.empty_like(inp.x)
    api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, None, ws,
                    route_state=inp.route_state)          # one-time set-up outside the count
    torch.cuda.synchronize()
    n0 = api.kernel_launches()
    api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, None, ws,
                    route_state=inp.route_state)
    n1 = api.kernel_launches()
    torch.cuda.synchronize()
    api.moe_check_device_errors(ws)
    assert n1 - n0 == expected
