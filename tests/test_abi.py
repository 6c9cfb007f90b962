"""The C-ABI library loads, exports every entry point include/moe.h declares,
and validates arguments on the host (no GPU needed: validation returns
before any CUDA call)."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from mixture_experts_layer_63_b200 import build
    build.build()
    return api.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 10
    assert set(names) == set(api.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_struct_sizes(L):
    assert ctypes.sizeof(api.MoeConfig) == 88
    assert ctypes.sizeof(api.MoeSizes) == 64


def test_struct_layout_matches_the_header(tmp_path):
    """Every field offset of the ctypes structs equals the C compiler's
    offsetof on include/moe.h (gcc, host only)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe.h"', 'int main(void) {']
    for st, cname in ((api.MoeConfig, "moe_config"), (api.MoeSizes, "moe_sizes")):
        lines.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in st._fields_:
            lines.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = dict(l.split() for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                  check=True).stdout.splitlines())
    for st, cname in ((api.MoeConfig, "moe_config"), (api.MoeSizes, "moe_sizes")):
        assert int(got[cname]) == ctypes.sizeof(st)
        for f, _ in st._fields_:
            assert int(got[f"{cname}.{f}"]) == getattr(st, f).offset, f


def test_launch_counter_reads_without_a_gpu(L):
    n = api.kernel_launches()
    assert n >= 0
    # a call that fails host validation launches nothing
    with pytest.raises(api.MoeError):
        api.query_sizes(_cfg(T=0))
    assert api.kernel_launches() == n


def test_status_strings(L):
    for s in range(7):
        assert api.status_string(s)
    assert api.status_string(99) == "unknown status"


def test_sizes_of_the_workloads(L):
    for name, w in WORKLOADS.items():
        s = api.query_sizes(api.config_from_workload(w))
        if w.mode == "ec":
            assert s.rows_cap == w.E * w.ec_capacity and s.tok_rows_len == w.E * w.T
        else:
            assert s.rows_cap == w.T * w.k and s.tok_rows_len == w.T * w.k
        assert s.rows_total == s.rows_cap + w.S * w.T
        assert s.workspace >= s.step_workspace >= 256
        es = 4 if w.dtype == "f32" else 2
        assert s.host_workspace >= s.workspace + 2 * w.T * w.d_model * es


def _cfg(**kw):
    c = api.config_from_workload(WORKLOADS["gshard"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status", [
    ("T", 0, api.MOE_ERR_INVALID_ARG),
    ("k", 0, api.MOE_ERR_INVALID_ARG),
    ("k", 17, api.MOE_ERR_INVALID_ARG),
    ("k", 9, api.MOE_ERR_UNSUPPORTED),
    ("E", 300, api.MOE_ERR_UNSUPPORTED),
    ("d_model", 100, api.MOE_ERR_UNSUPPORTED),
    ("d_ff", 96, api.MOE_ERR_UNSUPPORTED),
    ("dtype", 7, api.MOE_ERR_INVALID_ARG),
    ("act", 3, api.MOE_ERR_INVALID_ARG),
    ("S", 9, api.MOE_ERR_UNSUPPORTED),
    ("n_groups", 3, api.MOE_ERR_INVALID_ARG),       # 16 experts do not split into 3 groups
    ("keep_den", 10, api.MOE_ERR_INVALID_ARG),      # capacity and keep-fraction together
    ("route_rule", 5, api.MOE_ERR_INVALID_ARG),
    ("reserved", 1, api.MOE_ERR_INVALID_ARG),
    ("local_groups", 3, api.MOE_ERR_INVALID_ARG),   # 4096 tokens do not split into 3 groups
    ("local_groups", 256, api.MOE_ERR_UNSUPPORTED), # groups of 16 tokens: below one 32-token unit
    ("local_groups", -1, api.MOE_ERR_INVALID_ARG),
    ("capacity_factor", float("nan"), api.MOE_ERR_INVALID_ARG),
    ("capacity_factor", float("inf"), api.MOE_ERR_INVALID_ARG),
])
def test_invalid_configs_rejected(L, field, value, status):
    c = _cfg(**{field: value})
    with pytest.raises(api.MoeError) as ei:
        api.query_sizes(c)
    assert ei.value.status == status


def test_group_limit_needs_enough_experts(L):
    c = _cfg(n_groups=8, topk_groups=1, k=2, capacity_factor=0.0)   # 1 group of 2 experts holds k=2: ok
    api.query_sizes(c)
    c = _cfg(n_groups=8, topk_groups=1, k=3, capacity_factor=0.0)
    with pytest.raises(api.MoeError):
        api.query_sizes(c)


def test_expert_choice_options(L):
    w = WORKLOADS["deepseekmoe_ec"]
    c = api.config_from_workload(w)
    api.query_sizes(c)
    c.ec_capacity = w.T + 1
    with pytest.raises(api.MoeError):
        api.query_sizes(c)
    c = api.config_from_workload(w)
    c.route_rule = api.MOE_ROUTE_LOAD                # routing rules are token-choice options
    with pytest.raises(api.MoeError):
        api.query_sizes(c)


def test_local_groups_need_a_capacity(L):
    c = _cfg(local_groups=4)
    api.query_sizes(c)
    c = _cfg(local_groups=4, capacity_factor=0.0)
    with pytest.raises(api.MoeError):
        api.query_sizes(c)


def test_null_pointers_rejected_before_any_launch(L):
    """Host validation returns before touching CUDA, so this runs without a GPU."""
    c = _cfg()
    s = api.query_sizes(c)
    f = L.moe_route
    st = f(ctypes.byref(c), None, None, None, None, None, None, None, None, None, 0, None)
    assert st == api.MOE_ERR_INVALID_ARG
    # workspace too small
    buf = ctypes.create_string_buffer(4096 + 256)
    addr = (ctypes.addressof(buf) + 255) & ~255
    st = L.moe_forward(ctypes.byref(c), 16, 16, None, None, 16, None, 16, 16, None, addr, 1024, None)
    assert st == api.MOE_ERR_WORKSPACE
    # misaligned workspace
    st = L.moe_forward(ctypes.byref(c), 16, 16, None, None, 16, None, 16, 16, None, addr + 8,
                       s.workspace, None)
    assert st == api.MOE_ERR_INVALID_ARG
    # a routing rule that reads route_state, without one
    c2 = _cfg(T=64, d_model=64, d_ff=64, capacity_factor=1.0)
    c2.route_rule = api.MOE_ROUTE_BIAS
    ws = ctypes.create_string_buffer(api.query_sizes(c2).workspace + 256)
    wa = (ctypes.addressof(ws) + 255) & ~255
    st = L.moe_forward(ctypes.byref(c2), 16, 16, None, None, 16, None, 16, 16, None, wa,
                       api.query_sizes(c2).workspace, None)
    assert st == api.MOE_ERR_INVALID_ARG
    st = L.moe_route_bias_update(ctypes.byref(c2), None, None, 0.001, None)
    assert st == api.MOE_ERR_INVALID_ARG
    st = L.moe_combine(ctypes.byref(c), None, None, None, None)
    assert st == api.MOE_ERR_INVALID_ARG


def test_cpu_tensors_refused(L):
    import torch
    c = _cfg()
    x = torch.zeros(c.T, c.d_model, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.moe_combine(c, x, x, x)


def _lib_capacity(w, T=None, cf=None):
    c = api.config_from_workload(w, T)
    if cf is not None:
        c.capacity_factor = cf
    return api.query_sizes(c).capacity


def test_library_capacity_matches_the_oracle(L):
    """The expert capacity the library derives from capacity_factor (GShard
    section 1: C = O(N/E), per local group with group dispatching) equals the
    oracle's ceil(cf * k * T / E) for the fp32 factor, clamped to the tokens
    of a group."""
    import numpy as np
    from dataclasses import replace

    from oracle import moe_oracle as O

    def oracle_c(T, E, k, cf):
        return min(O.capacity_from_factor(T, E, k, float(np.float32(cf))), T)

    tiny, gshard, local = WORKLOADS["tiny_f32"], WORKLOADS["gshard"], WORKLOADS["gshard_local"]
    assert _lib_capacity(tiny) == oracle_c(256, 8, 2, 1.25) == 80
    assert _lib_capacity(gshard) == oracle_c(4096, 16, 2, 1.25) == 640
    G = local.local_groups
    assert _lib_capacity(local) == oracle_c(4096 // G, 16, 2, 1.25) == 160
    # factor 1, top-2: 2N/(G*E) per group (GShard's local-group capacity)
    assert _lib_capacity(replace(local, capacity_factor=1.0)) == 2 * 4096 // (G * 16)
    # factors whose product is not an integer, or not exact in binary
    rng = np.random.default_rng(5)
    for cf in [0.1, 0.3, 1.1, 1.3, 2.7, 1e-3, 1e-30, 7.0, 100.0, 3e9]:
        for T in (96, 1000, 4096):
            w = replace(gshard, T=T, capacity_factor=cf)
            assert _lib_capacity(w) == oracle_c(T, 16, 2, cf), (cf, T)
    for _ in range(200):
        T, E = int(rng.integers(1, 5000)), int(rng.integers(1, 257))
        k = int(rng.integers(1, min(E, 8) + 1))
        cf = float(np.float32(rng.uniform(0.01, 4.0)))
        w = replace(gshard, T=T, E=E, k=k, capacity_factor=cf)
        assert _lib_capacity(w) == oracle_c(T, E, k, cf), (T, E, k, cf)
    # no capacity: 0; expert choice: 0 (its C is ec_capacity)
    assert _lib_capacity(replace(gshard, capacity_factor=0.0)) == 0
    assert _lib_capacity(WORKLOADS["deepseekmoe_ec"]) == 0


def test_permute_workspace_is_the_permutation_share(L):
    """moe_sizes.permute_workspace: the scratch moe_permute uses (what
    moe_permute_noalloc needs in its fixed array), within step_workspace."""
    for name, w in WORKLOADS.items():
        s = api.query_sizes(api.config_from_workload(w))
        assert 4096 <= s.permute_workspace <= s.step_workspace, name
    # the bf16 layers' step workspace holds the GEMMs' 24 MiB stream-K slab
    # as well, which the permutation does not use
    s = api.query_sizes(api.config_from_workload(WORKLOADS["gshard"]))
    assert s.step_workspace - s.permute_workspace >= 24 << 20


def test_new_entry_points_validate_on_the_host(L):
    """moe_forward_host refuses NULL host buffers and a workspace below
    host_workspace, moe_workspace_set_wait_limit a workspace below its 4 KiB
    control block: both before any CUDA call."""
    c = _cfg(T=64, d_model=64, d_ff=64)
    s = api.query_sizes(c)
    assert s.host_workspace > s.workspace
    buf = ctypes.create_string_buffer(s.host_workspace + 256)
    addr = (ctypes.addressof(buf) + 255) & ~255
    st = L.moe_forward_host(ctypes.byref(c), None, 16, None, None, 16, None, 16, None, None, addr,
                            s.host_workspace, None, None, None)
    assert st == api.MOE_ERR_INVALID_ARG
    st = L.moe_forward_host(ctypes.byref(c), 16, 16, None, None, 16, None, 16, 16, None, addr,
                            s.workspace, None, None, None)
    assert st == api.MOE_ERR_WORKSPACE
    assert L.moe_workspace_set_wait_limit(addr, 1024, 1000, None) == api.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_set_wait_limit(None, 1 << 20, 1000, None) == api.MOE_ERR_INVALID_ARG


def test_binding_checks_buffer_sizes():
    """A short output buffer is a Python error, not a write past its end
    (checked before the pointer is handed to the library)."""
    import torch
    c = _cfg(T=64, d_model=64, d_ff=64)
    n = api._Need(c)
    assert n.td == 64 * 64 and n.tok_rows == 64 * 2
    t = torch.empty(8)
    with pytest.raises(ValueError):
        api._ptr(t)                      # not a CUDA tensor
