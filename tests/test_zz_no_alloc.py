"""moe_permute_noalloc against moe_permute.

Some callers cannot allocate device memory: a plugin that a host program hands
only its input and output buffers, or a process that must keep a fixed device
footprint once it has started.  For them the library offers
moe_permute_noalloc, which takes its scratch from a fixed 8 MiB array compiled
into the library instead of a caller workspace; configurations whose
permutation scratch (moe_sizes.permute_workspace) exceeds it are refused.  Its outputs must equal
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


def _largest_ec_tokens_within_the_array():
    """Expert choice on 64 experts: the most tokens (a multiple of 32) whose
    permutation scratch (moe_sizes.permute_workspace, mostly the transposed
    probabilities, 64 * T * 4 bytes) still fits the fixed array."""
    T = api.NOALLOC_SCRATCH_BYTES // (64 * 4) // 32 * 32
    while api.query_sizes(api.config_from_workload(
            WORKLOADS["deepseekmoe_ec"].with_tokens(T))).permute_workspace > api.NOALLOC_SCRATCH_BYTES:
        T -= 32
    return T


def test_noalloc_limit_is_the_permutation_scratch():
    """The limit is moe_sizes.permute_workspace, not step_workspace (which also
    holds the GEMMs' stream-K slab): a configuration just under it runs and
    matches moe_permute on two calls in a row; 32 more tokens are refused."""
    T = _largest_ec_tokens_within_the_array()
    w = WORKLOADS["deepseekmoe_ec"].with_tokens(T)
    s = api.query_sizes(api.config_from_workload(w))
    assert api.NOALLOC_SCRATCH_BYTES - (64 << 10) < s.permute_workspace <= api.NOALLOC_SCRATCH_BYTES
    assert s.step_workspace > api.NOALLOC_SCRATCH_BYTES
    for seed in (23, 24):
        inp, cfg, B = _routing(w, seed)
        api.moe_permute(cfg, inp.x, None, None, B.probs, B.counts, B.offsets, B.tok_rows,
                        B.row_token, B.row_gate, B.x_perm, B.n_dropped, B.ws)
        torch.cuda.synchronize()
        R = int(B.offsets[w.E].item())
        ref = _outputs(B, R)
        for t in (B.counts, B.offsets, B.n_dropped, B.tok_rows, B.row_token, B.row_gate):
            t.fill_(-7)
        B.x_perm.zero_()
        api.moe_permute_noalloc(cfg, inp.x, None, None, B.probs, B.counts, B.offsets, B.tok_rows,
                                B.row_token, B.row_gate, B.x_perm, B.n_dropped)
        torch.cuda.synchronize()
        for a, b in zip(_outputs(B, R), ref):
            assert torch.equal(a, b)
    del inp, B
    # 32 more tokens: the transposed probabilities no longer fit
    w2 = WORKLOADS["deepseekmoe_ec"].with_tokens(T + 32)
    cfg2 = api.config_from_workload(w2)
    assert api.query_sizes(cfg2).permute_workspace > api.NOALLOC_SCRATCH_BYTES
    # refused by the library before it touches any buffer (the C call directly:
    # the binding's own size checks would refuse these stand-in pointers first)
    import ctypes
    st = api._noalloc()(ctypes.byref(cfg2), 256, None, None, 256, 256, 256, 256, 256, 256, 256, 256,
                        None)
    assert st == api.MOE_ERR_WORKSPACE
