"""api.HostPipeline: batches from pinned host memory through the layer with
overlapped copies give the same outputs, bit for bit, as one forward per
batch on resident tensors."""
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from tests.gpu_common import SMALL, gpu_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["gshard_s", "dsv2_s"])
def test_pipeline_matches_direct_forwards(name):
    w = SMALL[name]
    inp = gpu_inputs(w, seed=31, grid=False)
    cfg = api.config_from_workload(w)
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias,
                         route_state=inp.route_state)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    xs = [torch.randn(w.T, w.d_model, generator=g, device="cuda").to(inp.x.dtype) for _ in range(5)]
    want = [layer(x).clone() for x in xs]
    torch.cuda.synchronize()
    x_host = [x.cpu().pin_memory() for x in xs]
    y_host = [torch.empty_like(x).pin_memory() for x in x_host]
    pipe = api.HostPipeline(layer)
    for xh, yh in zip(x_host, y_host):
        pipe.submit(xh, yh)
    pipe.synchronize()
    for i, (yh, yw) in enumerate(zip(y_host, want)):
        assert torch.equal(yh, yw.cpu()), i
    api.moe_check_device_errors(layer.ws)
