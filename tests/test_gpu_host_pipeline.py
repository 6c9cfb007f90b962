"""moe_forward_host (the C-ABI call on host buffers) and api.HostPipeline
built on it: batches from pinned host memory through the layer, with copies
on their own streams overlapping the forwards and two workspaces in turn,
give the same outputs, bit for bit, as one forward per batch on resident
tensors; so does the plain call on one stream, pinned or pageable."""
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
    for ws in pipe.ws:
        api.moe_check_device_errors(ws)


@pytest.mark.parametrize("pinned", [True, False])
def test_forward_host_on_one_stream(pinned):
    w = SMALL["dsv2_s"]
    inp = gpu_inputs(w, seed=32, grid=False)
    cfg = api.config_from_workload(w)
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias)
    want = layer(inp.x).cpu()
    ws = api.new_workspace(cfg, host=True)
    xh = inp.x.cpu()
    yh = torch.full_like(xh, float("nan"))
    if pinned:
        xh, yh = xh.pin_memory(), yh.pin_memory()
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    for _ in range(2):                       # the second call reuses the workspace's events
        api.moe_forward_host(cfg, xh, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, yh, counts, ws)
        torch.cuda.synchronize()
        assert torch.equal(yh, want)
    assert torch.equal(counts, layer.counts)
    api.moe_check_device_errors(ws)


def test_forward_host_refuses_device_buffers_and_a_short_workspace():
    w = SMALL["gshard_s"]
    inp = gpu_inputs(w, seed=33, grid=False)
    cfg = api.config_from_workload(w)
    with pytest.raises(ValueError):
        api.moe_forward_host(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2,
                             inp.x.cpu(), None, api.new_workspace(cfg, host=True))
    with pytest.raises(api.MoeError) as ei:
        api.moe_forward_host(cfg, inp.x.cpu(), inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2,
                             inp.x.cpu(), None, api.new_workspace(cfg))
    assert ei.value.status == api.MOE_ERR_WORKSPACE
