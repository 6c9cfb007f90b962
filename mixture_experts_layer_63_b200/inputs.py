"""Seeded synthetic inputs for the sparse MoE FFN layer forward.

This module holds the five workload shapes and the random-number recipes
that produce their tensors.  It holds none of the layer's arithmetic: both
the CUDA path and the CPU oracle consume what it produces, and neither side
computes anything here.

Recipe (fixed draw order from one ``torch.Generator`` seeded with ``seed``):
``x`` [T, d], then ``w_router`` [E, d], then per expert (routed first, then
shared) ``w1`` [f, d], ``w3`` [f, d] (SwiGLU only), ``w2`` [d, f].  Values
are drawn in fp32 from N(0, 1) and scaled to the stated standard deviation,
then rounded to the workload dtype (bf16 round-to-nearest-even).

* ``x ~ N(0, 1)``.
* expert weights ``~ N(0, 1/fan_in)``: std ``d**-0.5`` for w1/w3 and
  ``f**-0.5`` for w2.
* router weights: std 0.02 where the workload states it (GShard-style),
  else ``d**-0.5``.
* Zipf-skewed routing (DeepSeekMoE-shaped workload): a fixed logit bias
  ``b_e = -s * ln(e + 1)``, expert 0 hottest.

``grid=True`` rounds ``x`` to multiples of 1/8 and the router weights to a
power-of-two grid of about 8-16 steps per standard deviation.  Every
product ``x_i * w_i`` is then a multiple of 2**-13 or finer and every
partial sum of a router dot product stays far below 2**24 of those steps,
so the fp32 router logits are exact whatever the summation order: the CUDA
router and the float64 oracle produce identical logits and therefore
identical routing.  Expert weights are never gridded.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and routing options of one MoE layer forward."""

    name: str
    T: int
    d_model: int
    E: int              # routed experts
    S: int              # shared (always-on) experts
    k: int              # experts per token (token choice)
    d_ff: int           # expert hidden size (d_ff, or d_moe for SwiGLU)
    act: str            # "relu" | "swiglu"
    dtype: str          # "f32" | "bf16"
    capacity_factor: float = 0.0      # <= 0: no capacity limit
    keep_num: int = 0                 # keep ceil(n_e * num / den) rows per expert
    keep_den: int = 0                 # 0/0: keep all
    mode: str = "tc"                  # "tc" token choice | "ec" expert choice
    ec_capacity: int = 0              # tokens per expert in expert-choice mode
    n_groups: int = 0                 # group-limited routing: groups of experts
    topk_groups: int = 0              # groups kept per token
    renormalize: bool = False         # gates divided by the sum of the selected p
    router_std: float | None = None   # None: d_model ** -0.5
    zipf_s: float = 0.0               # > 0: Zipf logit bias over experts
    route_rule: str = "softmax"       # selection keys: "softmax" | "bias" | "load"
    route_alpha: float = 0.0          # load-aware coefficient
    local_groups: int = 1             # GShard local groups (capacity per group)

    def with_tokens(self, T: int) -> "Workload":
        """Same layer on T tokens; expert choice keeps C = T * k / E."""
        if self.mode == "ec":
            return replace(self, T=T, ec_capacity=max(1, T * self.k // self.E))
        return replace(self, T=T)


WORKLOADS: dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", T=256, d_model=64, E=8, S=0, k=2, d_ff=128,
                         act="relu", dtype="f32", capacity_factor=1.25),
    "gshard": Workload("gshard", T=4096, d_model=1024, E=16, S=0, k=2, d_ff=4096,
                       act="relu", dtype="bf16", capacity_factor=1.25, router_std=0.02),
    "mixtral": Workload("mixtral", T=8192, d_model=4096, E=8, S=0, k=2, d_ff=14336,
                        act="swiglu", dtype="bf16", renormalize=True),
    "deepseekmoe_tc": Workload("deepseekmoe_tc", T=16384, d_model=2048, E=64, S=2, k=6,
                               d_ff=1408, act="swiglu", dtype="bf16", zipf_s=1.1),
    "deepseekmoe_ec": Workload("deepseekmoe_ec", T=16384, d_model=2048, E=64, S=2, k=6,
                               d_ff=1408, act="swiglu", dtype="bf16", zipf_s=1.1,
                               mode="ec", ec_capacity=16384 * 6 // 64),
    "deepseek_v2": Workload("deepseek_v2", T=8192, d_model=5120, E=160, S=2, k=6,
                            d_ff=1536, act="swiglu", dtype="bf16", n_groups=8,
                            topk_groups=3, keep_num=9, keep_den=10),
    # DeepSeek-V3's routing on the pages: 256 routed + 1 shared experts, top-8,
    # at most 4 of 8 nodes (groups) per token, auxiliary-loss-free bias routing.
    # The pages give no V3 hidden sizes: DeepSeek-V2's (5120 / 1536) stand in.
    "deepseek_v3": Workload("deepseek_v3", T=8192, d_model=5120, E=256, S=1, k=8,
                            d_ff=1536, act="swiglu", dtype="bf16", n_groups=8,
                            topk_groups=4, route_rule="bias"),
    # GShard with local group dispatching: 4 groups of 1024 tokens
    "gshard_local": Workload("gshard_local", T=4096, d_model=1024, E=16, S=0, k=2, d_ff=4096,
                             act="relu", dtype="bf16", capacity_factor=1.25, router_std=0.02,
                             local_groups=4),
}


@dataclass
class LayerInputs:
    """One seeded set of layer inputs (torch tensors on one device)."""

    x: torch.Tensor                 # [T, d]
    w_router: torch.Tensor          # [E, d]
    bias: torch.Tensor | None       # [E] fp32 or None
    w1: torch.Tensor                # [E+S, f, d]
    w3: torch.Tensor | None         # [E+S, f, d] (SwiGLU) or None
    w2: torch.Tensor                # [E+S, d, f]
    route_state: torch.Tensor | None = None   # [E] fp32: routing bias or utilisation


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _router_grid_step(std: float) -> float:
    # a power of two giving 8..16 grid steps per standard deviation
    return 2.0 ** -(math.ceil(math.log2(1.0 / std)) + 3)


def make_inputs(w: Workload, seed: int = 0, device: str | torch.device = "cpu",
                grid: bool = False, with_weights: bool = True) -> LayerInputs:
    """Draw the workload's tensors in the fixed order documented above."""
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dt = torch_dtype(w)
    T, d, E, S, f = w.T, w.d_model, w.E, w.S, w.d_ff

    x = torch.randn(T, d, generator=g, device=dev, dtype=torch.float32)
    if grid:
        x = torch.clamp(torch.round(x * 8.0) / 8.0, -7.875, 7.875)
    x = x.to(dt)

    r_std = w.router_std if w.router_std is not None else d ** -0.5
    w_router = torch.randn(E, d, generator=g, device=dev, dtype=torch.float32) * r_std
    if grid:
        step = _router_grid_step(r_std)
        lim = 8.0 * r_std
        w_router = torch.round(torch.clamp(w_router, -lim, lim) / step) * step
    w_router = w_router.to(dt)

    bias = None
    if w.zipf_s > 0:
        b64 = torch.tensor([-w.zipf_s * math.log(e + 1.0) for e in range(E)], dtype=torch.float64)
        bias = b64.to(torch.float32).to(dev)

    state = route_state(w, seed, dev, grid)
    if not with_weights:
        return LayerInputs(x, w_router, bias, None, None, None, state)

    G = E + S
    w1 = torch.empty(G, f, d, device=dev, dtype=dt)
    w3 = torch.empty(G, f, d, device=dev, dtype=dt) if w.act == "swiglu" else None
    w2 = torch.empty(G, d, f, device=dev, dtype=dt)
    s_in, s_hid = d ** -0.5, f ** -0.5
    for e in range(G):
        w1[e] = (torch.randn(f, d, generator=g, device=dev, dtype=torch.float32) * s_in).to(dt)
        if w3 is not None:
            w3[e] = (torch.randn(f, d, generator=g, device=dev, dtype=torch.float32) * s_in).to(dt)
        w2[e] = (torch.randn(d, f, generator=g, device=dev, dtype=torch.float32) * s_hid).to(dt)
    return LayerInputs(x, w_router, bias, w1, w3, w2, state)


def route_state(w: Workload, seed: int, device, grid: bool = False) -> torch.Tensor | None:
    """The per-expert routing state of the workload's rule, from a generator
    of its own (seed + 7919), so the other draws do not move.

    bias: b_e ~ N(0, (0.5 / E)^2), the scale of a softmax probability's
          spread over E experts, as a bias that has been trained for a while
          would be; grid: rounded to multiples of 2^-16.
    load: u_e ~ U(0, 1), a utilisation; grid: multiples of 1/16.
    """
    if w.route_rule == "softmax":
        return None
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 7919)
    if w.route_rule == "bias":
        st = torch.randn(w.E, generator=g, dtype=torch.float64) * (0.5 / w.E)
        if grid:
            st = torch.round(st * 65536.0) / 65536.0
    else:
        st = torch.rand(w.E, generator=g, dtype=torch.float64)
        if grid:
            st = torch.round(st * 16.0) / 16.0
    return st.to(torch.float32).to(device)


def router_sum_bound(inp: LayerInputs) -> float:
    """Largest sum_i |x_i * w_i| over all (token, expert) pairs, in float64.

    With ``grid=True`` inputs every partial sum of a router dot product is
    bounded by this value; it must stay below 2**10 for the fp32 logits to
    be exact (products are multiples of 2**-13 or coarser, so sums below
    2**10 need at most 23 significant bits).
    """
    xa = inp.x.double().abs()
    wa = inp.w_router.double().abs()
    return float((xa @ wa.T).max())
