"""moe_permute_noalloc against moe_permute.

Some callers cannot allocate device memory: a plugin that a host program hands
only its input and output buffers, or a process that must keep a fixed device
footprint once it has started.  For them the library offers
moe_permute_noalloc, which takes its scratch from a fixed 8 MiB array compiled
into the library instead of a caller workspace.  Its outputs must equal
moe_permute's bit for bit (all of them are integers, or copies), on two calls
in a row, because the shared array keeps the previous call's contents.

This file is collected last (its name sorts after the others), so a run that
stops at the first failure has already run every other test; it also passes
when run alone in a fresh process.
"""
import pytest
import torch

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = ["gshard", "deepseek_v2", "deepseekmoe_ec"]    # capacity, keep-fraction, expert choice


def _routing(w, seed):
    inp = make_inputs(w, seed=seed, device="cuda", grid=False, with_weights=False)
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    api.moe_route(cfg, inp.x, inp.w_router, inp.bias, B.logits, B.probs, B.topk_idx, B.topk_gate,
                  B.ws)
    return inp, cfg, B


def _outputs(B, R):
    return [B.counts.clone(), B.offsets.clone(), B.n_dropped.clone(), B.tok_rows.clone(),
            B.row_token[:R].clone(), B.row_gate[:R].clone(), B.x_perm[:R].clone()]


@pytest.mark.parametrize("name", CASES)
def test_noalloc_matches_workspace_permute_twice(name):
    assert torch.cuda.is_available()
    w = WORKLOADS[name]
    for seed in (21, 22):                        # two calls in a row, different routing
        inp, cfg, B = _routing(w, seed)
        api.moe_permute(cfg, inp.x, B.topk_idx, B.topk_gate, B.probs, B.counts, B.offsets,
                        B.tok_rows, B.row_token, B.row_gate, B.x_perm, B.n_dropped, B.ws)
        torch.cuda.synchronize()
        R = int(B.offsets[w.E].item())
        ref = _outputs(B, R)
        for t in (B.counts, B.offsets, B.n_dropped, B.tok_rows, B.row_token, B.row_gate):
            t.fill_(-7)
        B.x_perm.zero_()
        api.moe_permute_noalloc(cfg, inp.x, B.topk_idx, B.topk_gate, B.probs, B.counts, B.offsets,
                                B.tok_rows, B.row_token, B.row_gate, B.x_perm, B.n_dropped)
        torch.cuda.synchronize()
        got = _outputs(B, R)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    api.moe_check_device_errors(B.ws)


def test_noalloc_rejects_configurations_beyond_its_scratch():
    # expert choice on 65536 tokens x 64 experts needs 16 MiB of scratch for the
    # transposed probabilities: more than the fixed array holds
    w = WORKLOADS["deepseekmoe_ec"].with_tokens(65536)
    cfg = api.config_from_workload(w)
    assert api.query_sizes(cfg).step_workspace > api.NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    with pytest.raises(api.MoeError) as ei:
        api.moe_permute_noalloc(cfg, dummy, None, None, dummy, dummy, dummy, dummy, dummy,
                                dummy.float(), dummy, dummy)
    assert ei.value.status == api.MOE_ERR_WORKSPACE
