"""Helpers shared by the GPU parity tests: oracle configuration from a
workload, tensor <-> numpy conversion, the output tolerance rule."""
from __future__ import annotations

from dataclasses import replace

import numpy as np
import torch

from mixture_experts_layer_63_b200 import api
from mixture_experts_layer_63_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import moe_oracle as O

# Output tolerance: max |y - y_ref| <= TOL * rms(y_ref) + half an ulp of
# y_ref in the output format.  bf16: 2e-2, fp32: 1e-4 (read as relative to
# rms).  The half-ulp term is the storage rounding of the output itself: a
# bf16 value carries up to 2**-8 |y| of it, so without the term even the
# correctly rounded exact answer would break the rule wherever |y| > 5.12 rms.
TOL = {"bf16": 2e-2, "f32": 1e-4}
SIG_BITS = {"bf16": 8, "f32": 24}


def half_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    """Half an ulp of each |ref| in the output format (8 or 24 significant bits)."""
    _, e = np.frexp(np.abs(ref))                 # |ref| = m * 2**e, m in [0.5, 1)
    return np.ldexp(1.0, e - 1 - SIG_BITS[dtype])

# Shape-reduced versions of the five workloads: same routing options, sizes
# the oracle evaluates in seconds, several M tiles, ragged tails and partial
# N tiles (d or f not a multiple of 256 / 128).
SMALL = {
    "tiny_f32": WORKLOADS["tiny_f32"],
    "gshard_s": replace(WORKLOADS["gshard"], T=700, d_model=256, d_ff=320),
    "mixtral_s": replace(WORKLOADS["mixtral"], T=600, d_model=320, d_ff=192),
    "dsmoe_tc_s": replace(WORKLOADS["deepseekmoe_tc"], T=1000, d_model=256, d_ff=128),
    "dsmoe_ec_s": replace(WORKLOADS["deepseekmoe_ec"], T=1000, d_model=256, d_ff=128,
                          ec_capacity=1000 * 6 // 64),
    "dsv2_s": replace(WORKLOADS["deepseek_v2"], T=900, d_model=320, d_ff=192),
    # >= 1024 rows per expert: the up/down projections run on CTA pairs
    # (256-row tiles); ragged M tails, partial N tiles, shared experts
    "pair_relu_s": replace(WORKLOADS["gshard"], T=2100, E=4, d_model=256, d_ff=320),
    "pair_swiglu_s": replace(WORKLOADS["deepseekmoe_tc"], T=1400, E=8, k=6, d_model=320, d_ff=192),
    # CTA pairs, ReLU with a shared expert: last M-tiles of 24-31 rows (the
    # even CTA's rows only) and of 122 rows (both CTAs), the shared expert's
    # 2150 = 8 * 256 + 102 rows
    "pair_half_s": replace(WORKLOADS["gshard"], T=2150, E=4, S=1, d_model=256, d_ff=320),
    # one routed and one shared row a token: moe_forward adds both into y from
    # the down-projection (the folded combine), with single CTAs and with pairs
    "fold_shared_s": replace(WORKLOADS["gshard"], T=700, k=1, S=1, d_model=256, d_ff=320),
    "fold_shared_pair_s": replace(WORKLOADS["gshard"], T=2100, E=4, k=1, S=1, d_model=256, d_ff=320),
    # routing variants: DeepSeek-V3 bias routing (256 + 1 experts, top-8 of 4
    # groups), load-aware top-k, GShard local groups
    "dsv3_s": replace(WORKLOADS["deepseek_v3"], T=600, d_model=256, d_ff=128),
    "load_aware_s": replace(WORKLOADS["gshard"], T=700, d_model=256, d_ff=320, route_rule="load",
                            route_alpha=0.75, capacity_factor=0.0),
    "local_groups_s": replace(WORKLOADS["gshard_local"], T=768, d_model=256, d_ff=320),
    # 64 experts, two rows a token: the router GEMM's epilogue gates and zeroes
    # y, the down-projection adds the rows into it (folded combine)
    "fold_tc_s": replace(WORKLOADS["gshard"], T=700, E=64, d_model=256, d_ff=320),
}


def oracle_config(w: Workload) -> O.OracleConfig:
    cf = float(np.float32(w.capacity_factor))       # the fp32 factor the library takes
    Tg = w.T // max(1, w.local_groups)              # capacity of one expert in one group
    cap = min(O.capacity_from_factor(Tg, w.E, w.k, cf), Tg) if w.mode == "tc" else 0
    return O.OracleConfig(E=w.E, S=w.S, k=w.k, act=w.act, mode=w.mode, capacity=cap,
                          keep_num=w.keep_num, keep_den=w.keep_den,
                          ec_capacity=w.ec_capacity if w.mode == "ec" else 0,
                          n_groups=w.n_groups, topk_groups=w.topk_groups,
                          renormalize=w.renormalize, rule=w.route_rule,
                          alpha=float(np.float32(w.route_alpha)), local_groups=w.local_groups)


def to_np(t: torch.Tensor) -> np.ndarray:
    """Host numpy copy; bf16 becomes its uint16 bit pattern (the oracle's input form)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


class LazyExperts:
    """Expert weights fetched from the device one expert at a time (the
    oracle indexes w[e]); keeps host memory small for the large workloads."""

    def __init__(self, t: torch.Tensor | None):
        self.t = t
        self.cache: dict[int, np.ndarray] = {}

    def __getitem__(self, e: int):
        if self.t is None:
            return None
        e = int(e)
        if e not in self.cache:
            self.cache[e] = to_np(self.t[e])
        return self.cache[e]


def assert_close_rms(y: np.ndarray, ref: np.ndarray, dtype: str, what: str = "y"):
    """max over elements of (|y - ref| - half_ulp(ref)) <= TOL[dtype] * rms(ref)."""
    ref = ref.astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    diff = np.abs(y.astype(np.float64) - ref)
    excess = float(np.max(diff - half_ulp(ref, dtype)))
    tol = TOL[dtype]
    assert excess <= tol * rms, (f"{what}: max(|err| - half ulp) {excess:.3e} > {tol} * rms "
                                 f"{rms:.3e} (plain max|err| {diff.max():.3e})")
    return float(diff.max()) / rms


def round_to_format(ref: np.ndarray, dtype: str) -> np.ndarray:
    """ref rounded once, to nearest even, to the output format (bf16 or fp32)."""
    r32 = ref.astype(np.float32)
    if dtype == "f32":
        return r32.astype(np.float64)
    return torch.from_numpy(r32).to(torch.bfloat16).double().numpy()


def output_margins(y: np.ndarray, ref: np.ndarray, dtype: str) -> dict:
    """How close an output is to the oracle, relative to rms(ref):
    excess_over_rms         max(|y - ref| - half an ulp of ref) / rms, the
                            quantity the tolerance rule bounds (P17);
    plain_over_rms          max |y - ref| / rms;
    vs_rounded_ref_over_rms max(|y - r| - ulp(ref)) / rms with r = ref rounded
                            once to the output format: y may sit on the
                            neighbouring representable value of r, no further;
    identical_to_rounded    share of elements equal to r bit for bit."""
    ref = ref.astype(np.float64)
    y = y.astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    hu = half_ulp(ref, dtype)
    r = round_to_format(ref, dtype)
    return {"excess_over_rms": float(np.max(np.abs(y - ref) - hu)) / rms,
            "plain_over_rms": float(np.max(np.abs(y - ref))) / rms,
            "vs_rounded_ref_over_rms": float(np.max(np.abs(y - r) - 2 * hu)) / rms,
            "identical_to_rounded": float(np.mean(y == r)),
            "tol": TOL[dtype]}


def record_margin(case: str, m: dict) -> None:
    """Append the margins of one case as a JSON line to the file named by
    MOE_MARGIN_LOG (if set), for the design notes' tolerance table."""
    import json
    import os
    path = os.environ.get("MOE_MARGIN_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, **m}) + "\n")


def gpu_inputs(w: Workload, seed: int = 0, grid: bool = True):
    return make_inputs(w, seed=seed, device="cuda", grid=grid)


def state_dev(inp):
    """The routing state of the inputs on the GPU (or None)."""
    return None if inp.route_state is None else inp.route_state.cuda()


def state_np(inp):
    """The routing state of the inputs as a host fp32 array (or None)."""
    return None if inp.route_state is None else inp.route_state.detach().cpu().numpy()
