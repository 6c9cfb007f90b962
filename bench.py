#!/usr/bin/env python
"""Benchmark of the MoE FFN layer forward on B200 (tokens/s).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gshard] [--impl ours|reference]

One step = one whole forward of the layer (router, gate, selection,
permutation, expert FFNs, combine) over one batch of T tokens, inputs resident
in HBM.  The timed loop calls moe_forward_timed (the launches of moe_forward,
with CUDA events recorded at its phase boundaries on the launching stream);
L2 is flushed before every step, untimed: a 256 MB memset, then a read of
another 256 MB buffer, so the step starts with none of its data in L2 and
no dirty lines of the memset still to be written back to DRAM.  `e2e` times moe_forward through the public
layer object with the host->device copy of x and the device->host copy of y
inside the timed region (no flush there: every step streams all expert
weights, more than the 126 MB L2, and x arrives fresh from the host).  With N > 1 (torchrun), every rank runs its own
replica on its own tokens (no collective in the forward: weak scaling); the
time is the maximum over ranks.

`--impl reference` times the CPU oracle (the only reference this layer has)
on a bounded sample of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_63_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200; grouped-GEMM % bf16 peak; permute GB/s"
# the largest of the five layers (DeepSeek-V2-shaped: 160 + 2 experts, 7.6 GB
# of expert weights); --workload selects the others
DEFAULT_WORKLOAD = "deepseek_v2"
# expert GEMMs at least this long a step are held to the sustained tensor peak
SUSTAINED_MIN_MS = 1.0

# DRAM bytes (read + write) of the two expert GEMMs of one forward, from an
# ncu capture of the same kernels, with the sha256 (first 16 hex digits) of
# the GEMM sources (the kernel file, then its PTX wrappers) they were taken
# at; reported only while the sources are unchanged (null otherwise).
NCU_TRAFFIC: dict[str, dict] = {
    # up 151.11 + 40.05 MB, down 220.19 + 6.10 MB
    "gshard": {"bytes": 417_442_304, "src": "1f89c012e2ab7a21"},
    # captured on a 40 + 2-expert cut of the layer (15173 kept rows): up
    # 1496.68 + 40.32 MB, down 707.72 + 119.18 MB; scaled to the whole layer
    # as every expert's weights read once (7644 MB) plus the cut's other
    # bytes (382.1 MB) times the kept rows' ratio (60693 / 15173)
    "deepseek_v2": {"bytes": 9_172_527_711, "src": "1f89c012e2ab7a21"},
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _describe(w) -> str:
    s = (f"{w.name}: T={w.T} d_model={w.d_model} E={w.E}+{w.S}shared k={w.k} "
         f"{'SwiGLU' if w.act == 'swiglu' else 'ReLU'} d_ff={w.d_ff} {w.dtype}")
    if w.capacity_factor > 0:
        s += f" capacity_factor={w.capacity_factor}"
    if w.keep_den > 0:
        s += f" keep={w.keep_num}/{w.keep_den}"
    if w.mode == "ec":
        s += f" expert-choice C={w.ec_capacity}"
    if w.n_groups > 0:
        s += f" groups={w.topk_groups}of{w.n_groups}"
    if w.renormalize:
        s += " renormalized"
    if w.zipf_s > 0:
        s += f" zipf_bias={w.zipf_s}"
    return s


def _src_hash(*names: str) -> str:
    h = hashlib.sha256()
    for name in names:
        h.update(open(os.path.join(ROOT, "mixture_experts_layer_63_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    Reads NVML (what nvidia-smi reports) from a background thread every 2 ms,
    falling back to an `nvidia-smi -lms 200` process.  Reading only: no
    setting of the GPU is touched."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int, period_s: float = 0.002):
        import threading
        self.samples, self.proc, self.nvml, self.thread = [], None, None, None
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.sel)
            self.stop_flag = threading.Event()

            def run():
                while not self.stop_flag.is_set():
                    sm = pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
                    why = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((sm, why))
                    time.sleep(period_s)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
        except Exception:
            self.nvml = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "200", "-i", self.sel],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None

    def stop(self) -> dict | None:
        if self.nvml is not None:
            self.stop_flag.set()
            self.thread.join(timeout=2)
            mx = self.nvml.nvmlDeviceGetMaxClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
            if not self.samples:
                return None
            reasons = sorted({n for _, why in self.samples for b, n in self.REASONS.items() if why & b})
            return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": mx,
                    "reasons": reasons, "samples": len(self.samples), "source": "nvml"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


class _DeviceExperts:
    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        if self.t is None:
            return None
        v = self.t[int(e)].detach().contiguous().cpu()
        return v.view(torch.int16).numpy().view(np.uint16) if v.dtype == torch.bfloat16 else v.numpy()


def _np_in(t):
    v = t.detach().contiguous().cpu()
    return v.view(torch.int16).numpy().view(np.uint16) if v.dtype == torch.bfloat16 else v.numpy()


class OracleTimer:
    """The CPU oracle on one workload: full routing of all T tokens, then the
    expert FFNs and combine of a sample of n tokens; tokens/s is extrapolated
    as T / (t_route + t_ffn * T / n)."""

    def __init__(self, w, seed: int, device: str):
        from oracle import moe_oracle as O
        self.O, self.w = O, w
        inp = make_inputs(w, seed=seed, device=device, grid=False)
        self.x = _np_in(inp.x)
        self.w_router = _np_in(inp.w_router)
        self.bias = None if inp.bias is None else _np_in(inp.bias)
        # expert weights widened per use, like the oracle's own tests do
        self.w1 = _DeviceExperts(inp.w1)
        self.w2 = _DeviceExperts(inp.w2)
        self.w3 = _DeviceExperts(inp.w3)
        Tg = w.T // max(1, w.local_groups)
        cf = float(np.float32(w.capacity_factor))
        cap = min(O.capacity_from_factor(Tg, w.E, w.k, cf), Tg) if w.mode == "tc" else 0
        self.state = None if inp.route_state is None else inp.route_state.cpu().numpy()
        self.cfg = O.OracleConfig(E=w.E, S=w.S, k=w.k, act=w.act, mode=w.mode, capacity=cap,
                                  keep_num=w.keep_num, keep_den=w.keep_den,
                                  ec_capacity=w.ec_capacity if w.mode == "ec" else 0,
                                  n_groups=w.n_groups, topk_groups=w.topk_groups,
                                  renormalize=w.renormalize, rule=w.route_rule,
                                  alpha=float(np.float32(w.route_alpha)),
                                  local_groups=w.local_groups)

    def step(self, n: int, rng) -> tuple[float, float, float]:
        O = self.O
        t0 = time.perf_counter()
        logits = O.router_logits(self.x, self.w_router, self.bias)
        _, _, _, disp = O.route(self.cfg, logits, self.state)
        t1 = time.perf_counter()
        toks = np.sort(rng.choice(self.w.T, size=min(n, self.w.T), replace=False))
        O.combine_tokens(self.cfg, self.x, self.w1, self.w2, self.w3, disp, toks)
        t2 = time.perf_counter()
        t_route, t_ffn = t1 - t0, t2 - t1
        est = t_route + t_ffn * self.w.T / len(toks)
        return self.w.T / est, t_route, t_ffn

    def calibrate(self, budget_s: float) -> int:
        """Largest power-of-two sample whose FFN part stays near budget_s."""
        rng = np.random.default_rng(0)
        n = 32
        while True:
            _, tr, tf = self.step(n, rng)
            if tf >= budget_s / 2 or n >= self.w.T:
                return n
            n = min(self.w.T, n * 2)


def cpu_baseline(w, seed: int, device: str, budget_s: float = 12.0) -> dict:
    ot = OracleTimer(w, seed, device)
    n = ot.calibrate(budget_s)
    rng = np.random.default_rng(1)
    v, tr, tf = ot.step(n, rng)
    return {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"routing of all {w.T} tokens ({tr:.2f} s) + expert FFNs and combine of "
                      f"{min(n, w.T)} sampled tokens ({tf:.2f} s), extrapolated to {w.T} tokens"}


def run_reference(args, w) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    ot = OracleTimer(w, args.seed, dev)
    n = ot.calibrate(3.0)
    rng = np.random.default_rng(2)
    for _ in range(args.warmup):
        ot.step(n, rng)
    vals, t0 = [], time.perf_counter()
    for _ in range(args.steps):
        vals.append(ot.step(n, rng)[0])
    elapsed = time.perf_counter() - t0
    v = float(statistics.mean(vals))
    sample = (f"per step: routing of all {w.T} tokens + expert FFNs/combine of {n} sampled "
              f"tokens, extrapolated to {w.T} tokens")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * w.T / v, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": _describe(w), "parallelism": "cpu oracle, rank 0 only"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": elapsed,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class L2Flush:
    """Evicts the step's data from L2: a 256 MB memset (larger than the 126 MB
    L2), then a read of a second 256 MB buffer, which leaves L2 holding clean
    lines of that buffer.  Without the read, the memset's dirty lines are
    written back to DRAM during the next step, at its expense."""

    def __init__(self, mb: int = 256):
        self.wr = torch.empty(mb * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.rd = torch.zeros(mb * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
        self.sink = torch.empty((), dtype=torch.float32, device="cuda")

    def __call__(self):
        self.wr.zero_()
        torch.sum(self.rd, dim=0, out=self.sink)


def run_ours(args, w) -> None:
    from mixture_experts_layer_63_b200 import api, replicas

    info = replicas.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    # replicas: same weights on every rank, each rank its own tokens
    inp = make_inputs(w, seed=args.seed, device="cuda", grid=False)
    if world > 1:
        g = torch.Generator(device="cuda")
        g.manual_seed(replicas.token_seed(args.seed, rank, world))
        inp.x = torch.randn(w.T, w.d_model, generator=g, device="cuda").to(inp.x.dtype)
    cfg = api.config_from_workload(w)
    sizes = api.query_sizes(cfg)
    ws = api.new_workspace(cfg)
    y = torch.empty_like(inp.x)
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    flush = L2Flush()
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is None:
            api.moe_forward(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y, counts, ws,
                            route_state=inp.route_state)
        else:
            api.moe_forward_timed(cfg, inp.x, inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2, y,
                                  counts, ws, ev, route_state=inp.route_state)

    def new_events(n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n)] for _ in range(args.steps)]
        for row in evs:                       # create the CUDA events before handing them over
            for ev in row:
                ev.record(stream)
        return evs

    for _ in range(args.warmup):
        flush()
        step()
    api.moe_check_device_errors(ws)
    # timed region: each step between two events on the launching stream; inside
    # the forward, events only around the expert FFN phase (the roofline kernels)
    evs = new_events(4)
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    launches0 = api.kernel_launches()
    for i in range(args.steps):
        flush()
        evs[i][0].record(stream)
        step([None, None, evs[i][1], evs[i][2], None])
        evs[i][3].record(stream)
    launches = api.kernel_launches() - launches0        # libmoe kernels in the timed region
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    api.moe_check_device_errors(ws)
    total_ms = replicas.max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in evs), dist, device="cuda")
    ffn_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_step = total_ms / args.steps
    value = replicas.throughput(world, w.T, args.steps, total_ms)

    # phase split (separate steps, not part of `value`): events at every phase
    # boundary, which also keeps each phase's kernels from overlapping the next
    pevs = new_events(5)
    for i in range(args.steps):
        flush()
        step(pevs[i])
    torch.cuda.synchronize()
    per = np.array([[pevs[i][j].elapsed_time(pevs[i][j + 1]) for j in range(4)]
                    for i in range(args.steps)])          # ms: route, permute, ffn, combine

    # algorithmic work of this batch: the kept routed rows, offsets[E] of the
    # same routing and permutation run once through the step entry points
    B = api.step_buffers(cfg)
    api.moe_route(cfg, inp.x, inp.w_router, inp.bias, B.logits, B.probs, B.topk_idx, B.topk_gate,
                  B.ws, route_state=inp.route_state)
    api.moe_permute(cfg, inp.x, B.topk_idx, B.topk_gate, B.probs, B.counts, B.offsets, B.tok_rows,
                    B.row_token, B.row_gate, B.x_perm, B.n_dropped, B.ws)
    R = int(B.offsets[w.E].item())
    del B
    es = 4 if w.dtype == "f32" else 2
    rows = R + w.S * w.T
    nmat = 3 if w.act == "swiglu" else 2
    gemm_flops = 2.0 * rows * w.d_model * w.d_ff * nmat
    permute_bytes = (w.T * w.d_model + R * w.d_model) * es
    combine_bytes = rows * w.d_model * es + w.T * w.d_model * es    # gated rows in, y out
    route_bytes = (w.T * w.d_model + w.E * w.d_model) * es + 2 * w.T * w.E * 4
    weight_bytes = (w.E + w.S) * w.d_ff * w.d_model * nmat * es
    # moe_forward folds the combine into the down-projection when a token has
    # at most two rows (bf16 token choice, k + S <= 2): no combine phase then
    folded = w.dtype == "bf16" and w.mode == "tc" and w.k + w.S <= 2
    mean = per.mean(axis=0)                                # ms per call
    hbm, tfl, tfl_sus, peak_src = _peaks()
    gemm_tflops = gemm_flops / (ffn_ms * 1e-3) / 1e12
    # which tensor peak: the expert GEMMs of a step that run for a
    # millisecond or more do so under the 1000 W power cap (SM clocks read
    # inside the kernel, against the global timer, fall from about 1.73 GHz to
    # 1.2-1.4 GHz within the DeepSeek-V2 up-projection), which is the regime
    # of the seconds-long sustained GEMM peak; shorter ones (the GShard
    # shape: 0.14 ms) run at the clocks of the burst peak
    sustained = tfl_sus is not None and ffn_ms >= SUSTAINED_MIN_MS
    peak = tfl_sus if sustained else tfl
    # the expert GEMMs' floor: their flops at the tensor peak, or streaming
    # every expert's weights once at the HBM peak, whichever is longer
    floor_ms = max(gemm_flops / (peak * 1e12), weight_bytes / (hbm * 1e9)) * 1e3
    h = _src_hash("gemm_sm100.cu", "sm100_ptx.cuh")
    tr = NCU_TRAFFIC.get(w.name)
    traffic = tr["bytes"] if tr and tr.get("src") == h else None

    # end to end through the C-ABI call on host buffers (moe_forward_host, via
    # api.HostPipeline): every step copies its batch of x from pinned host
    # memory and its y back; two workspaces in turn and copy streams of their
    # own let the copies of neighbouring steps overlap the forward.  No L2
    # flush: every step streams the expert weights (larger than the L2 on
    # every workload) and x arrives fresh from the host, as a caller sees it
    layer = api.MoELayer(cfg, inp.w_router, inp.w1, inp.w2, inp.w3, inp.bias,
                         route_state=inp.route_state)
    x_host = [inp.x.cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty_like(x_host[0]).pin_memory() for _ in range(2)]
    y_dev = torch.empty_like(inp.x)
    pipe = api.HostPipeline(layer)
    for i in range(args.warmup):
        pipe.submit(x_host[i & 1], y_host[i & 1])
    pipe.synchronize()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for i in range(args.steps):
        pipe.submit(x_host[i & 1], y_host[i & 1])
    pipe.s_out.wait_stream(pipe.s_in)
    pipe.s_out.wait_stream(pipe.s_comp)
    e1.record(pipe.s_out)
    pipe.synchronize()
    for pws in pipe.ws:
        api.moe_check_device_errors(pws)
    e2e_ms = replicas.max_over_ranks(e0.elapsed_time(e1), dist, device="cuda")
    if dist:
        dist.barrier()
    e2e_value = replicas.throughput(world, w.T, args.steps, e2e_ms)
    # the same calls one after the other on one stream (no overlap), for reference
    del pipe
    hws = api.new_workspace(cfg, host=True)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    seq_ms = 0.0
    for i in range(args.steps):
        s0.record(stream)
        api.moe_forward_host(cfg, x_host[i & 1], inp.w_router, inp.bias, inp.w1, inp.w3, inp.w2,
                             y_host[i & 1], None, hws, route_state=inp.route_state)
        s1.record(stream)
        torch.cuda.synchronize()
        seq_ms += s0.elapsed_time(s1)
    api.moe_check_device_errors(hws)
    del hws
    e2e_seq = replicas.throughput(world, w.T, args.steps,
                                  replicas.max_over_ranks(seq_ms, dist, device="cuda"))

    # training: forward + backward (moe_backward) per step, separate steps,
    # not part of `value`; every rank takes the same steps
    backward = None
    if w.dtype == "bf16" and not args.no_backward:
        g = torch.Generator(device="cuda")
        g.manual_seed(args.seed + 17)
        dy = torch.randn(w.T, w.d_model, generator=g, device="cuda").to(inp.x.dtype)
        for _ in range(args.warmup):
            flush()
            layer(inp.x, out=y_dev)
            layer.backward(inp.x, dy)
        bev = new_events(3)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        for i in range(args.steps):
            flush()
            bev[i][0].record(stream)
            layer(inp.x, out=y_dev)
            bev[i][1].record(stream)
            layer.backward(inp.x, dy)
            bev[i][2].record(stream)
        torch.cuda.synchronize()
        api.moe_check_device_errors(layer.ws)
        bw_ms = replicas.max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in bev), dist, device="cuda")
        fb_ms = replicas.max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in bev), dist, device="cuda")
        # flops of the backward's contractions: recompute of the pre-activations,
        # dH, dX, dW2, dW1 (| dW3), plus the router's dx and dW_r
        nb = (2 + 1 + 2 + 1 + 2) if w.act == "swiglu" else (1 + 1 + 1 + 1 + 1)
        bw_flops = 2.0 * rows * w.d_model * w.d_ff * nb + 2 * 2.0 * w.T * w.E * w.d_model
        backward = {"ms_per_step": bw_ms / args.steps,
                    "tokens_per_s_fwd_bwd": replicas.throughput(world, w.T, args.steps, fb_ms),
                    "achieved_tflops": bw_flops / (bw_ms / args.steps * 1e-3) / 1e12,
                    "algorithmic_flops": bw_flops,
                    "note": "moe_backward after moe_forward, routing held fixed; separate steps"}
        del layer.bws

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.seed, "cuda")

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if w.dtype == "f32" else "bf16",
            "data": "synthetic: x ~ N(0,1), expert weights ~ N(0,1/fan_in), random init, seeded",
            "config": {"workload": _describe(w), "T": w.T, "d_model": w.d_model, "E": w.E,
                       "S": w.S, "k": w.k, "d_ff": w.d_ff,
                       "parallelism": f"replicas x{world} (no collective in the forward)",
                       "l2": "flushed before every step (untimed): 256 MB memset, then a 256 MB read "
                             "of another buffer (the memset's dirty lines written back before the step)"},
            "roofline": {"bound": "tensor", "kernel": "grouped GEMM (up + down projections)",
                         "achieved": gemm_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": gemm_tflops / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'}"
                                        + (" (expert GEMMs of %.2f ms a step: power-capped clocks)" % ffn_ms
                                           if sustained else ""),
                         "algorithmic_flops": gemm_flops,
                         "frac_of_burst": gemm_tflops / tfl,
                         "frac_of_sustained": gemm_tflops / tfl_sus if tfl_sus else None,
                         "weight_bytes": weight_bytes,
                         "floor_ms": floor_ms, "floor_bound": "tensor" if gemm_flops / (peak * 1e12)
                         >= weight_bytes / (hbm * 1e9) else "hbm (weights)",
                         "frac_of_floor": floor_ms / ffn_ms},
            "steps_us": {"route": mean[0] * 1e3, "permute": mean[1] * 1e3,
                         "expert_ffn": mean[2] * 1e3, "combine": mean[3] * 1e3,
                         "expert_ffn_in_timed_region": ffn_ms * 1e3,
                         "combine_folded_into_down_gemm": folded,
                         "note": "phase split from separate steps with an event at every phase boundary"},
            "bandwidth_gbs": {"route": route_bytes / (mean[0] * 1e-3) / 1e9,
                              "permute": permute_bytes / (mean[1] * 1e-3) / 1e9,
                              "combine": None if folded else combine_bytes / (mean[3] * 1e-3) / 1e9,
                              "hbm_peak": hbm},
            "rows": {"routed_kept": R, "shared": w.S * w.T, "capacity_rows": sizes.rows_cap},
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(x_host[0].numel() * x_host[0].element_size()),
                    "d2h_bytes_per_step": int(y_host[0].numel() * y_host[0].element_size()),
                    "sequential_value": e2e_seq,
                    "l2": "not flushed: each step streams %.0f MB of expert weights (L2: 126 MB)"
                          % (weight_bytes / 1e6),
                    "note": "moe_forward_host (C ABI, host buffers) with two workspaces and copy "
                            "streams: each step's host copies overlap its neighbours' forwards"},
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
            "backward": backward,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def run_route_only(args, w) -> None:
    """The routing step alone (moe_route: router logits, softmax, group limit,
    top-k), L2 flushed before every call, timed with CUDA events: the
    number a profile of the router kernel refers to.  Algorithmic bytes: x
    and W_r read, logits and probabilities written (fp32), top-k written."""
    from mixture_experts_layer_63_b200 import api
    torch.cuda.set_device(0)
    inp = make_inputs(w, seed=args.seed, device="cuda", with_weights=False)
    cfg = api.config_from_workload(w)
    B = api.step_buffers(cfg)
    flush = L2Flush()

    def route():
        api.moe_route(cfg, inp.x, inp.w_router, inp.bias, B.logits, B.probs, B.topk_idx, B.topk_gate,
                      B.ws, route_state=inp.route_state)

    for _ in range(args.warmup):
        flush()
        route()
    torch.cuda.synchronize()
    api.moe_check_device_errors(B.ws)
    ts = []
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        route()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    api.moe_check_device_errors(B.ws)
    es = 4 if w.dtype == "f32" else 2
    k = w.k if w.mode == "tc" else 0
    nbytes = (w.T + w.E) * w.d_model * es + 2 * w.T * w.E * 4 + 2 * w.T * k * 4
    us = float(np.median(ts))
    hbm = _peaks()[0]
    print(json.dumps({"mode": "route-only", "workload": w.name, "steps": args.steps,
                      "route_us": round(us, 2), "route_gbs": round(nbytes / us / 1e3, 1),
                      "hbm_frac": round(nbytes / us / 1e3 / hbm, 3), "algorithmic_bytes": nbytes}))


def run_gemm_vs_library(args, w) -> None:
    """The expert GEMMs of this workload's shape, all rows on one expert (a
    dense problem), through moe_expert_ffn, next to torch.matmul (cuBLAS) on
    the same operands.  A yardstick for the kernels only: the library GEMM is
    never on the layer's path."""
    from mixture_experts_layer_63_b200 import api
    torch.cuda.set_device(0)
    R, d, f = w.T * w.k, w.d_model, w.d_ff
    c = api.MoeConfig()
    c.T, c.d_model, c.E, c.S, c.k, c.d_ff = R, d, 1, 0, 1, f
    c.act = api.MOE_ACT_SWIGLU if w.act == "swiglu" else api.MOE_ACT_RELU
    c.mode, c.dtype = api.MOE_TOKEN_CHOICE, api.MOE_BF16
    s = api.query_sizes(c)
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    x = torch.randn(R, d, generator=g, device="cuda").bfloat16()
    w1 = (torch.randn(1, f, d, generator=g, device="cuda") * d ** -0.5).bfloat16()
    w3 = (torch.randn(1, f, d, generator=g, device="cuda") * d ** -0.5).bfloat16() if w.act == "swiglu" else None
    w2 = (torch.randn(1, d, f, generator=g, device="cuda") * f ** -0.5).bfloat16()
    offsets = torch.tensor([0, R], dtype=torch.int32, device="cuda")
    gate = torch.ones(R, device="cuda")
    h = torch.empty(s.rows_total, f, device="cuda", dtype=torch.bfloat16)
    y = torch.empty(s.rows_total, d, device="cuda", dtype=torch.float32)
    ws = api.new_workspace(c, step_only=True)
    flush = L2Flush()

    def ours():
        api.moe_expert_ffn(c, x, x, offsets, gate, w1, w3, w2, h, y, ws)

    def lib():
        a = x @ w1[0].T
        hh = torch.relu(a) if w3 is None else torch.nn.functional.silu(a) * (x @ w3[0].T)
        return hh @ w2[0].T

    def timed(fn):
        for _ in range(args.warmup):
            flush()
            fn()
        t = 0.0
        for _ in range(args.steps):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            t += e0.elapsed_time(e1)
        return t / args.steps

    t_ours, t_lib = timed(ours), timed(lib)
    fl = 2.0 * R * d * f * (3 if w3 is not None else 2)
    print(json.dumps({"mode": "gemm-vs-library", "workload": _describe(w), "rows": R, "d_model": d,
                      "d_ff": f, "ours_us": t_ours * 1e3, "ours_tflops": fl / t_ours / 1e9,
                      "torch_matmul_us": t_lib * 1e3, "torch_matmul_tflops": fl / t_lib / 1e9,
                      "ratio": t_lib / t_ours, "l2": "flushed before every call"}), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the forward + backward measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm-vs-library", action="store_true",
                    help="time the expert GEMMs on this workload's dense shape next to torch.matmul")
    ap.add_argument("--route-only", action="store_true",
                    help="time the routing step (moe_route) alone on this workload")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling shape: this many tokens instead of the workload's")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling shape: this many routed experts instead of the workload's")
    ap.add_argument("--d-ff", type=int, default=0,
                    help="profiling shape: this expert hidden size instead of the workload's")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]
    if args.experts:
        from dataclasses import replace
        w = replace(w, E=args.experts, name=f"{w.name}[E={args.experts}]",
                    ec_capacity=w.T * w.k // args.experts if w.mode == "ec" else 0)
    if args.tokens:
        from dataclasses import replace
        w = replace(w.with_tokens(args.tokens), name=f"{w.name}[T={args.tokens}]")
    if args.d_ff:
        from dataclasses import replace
        w = replace(w, d_ff=args.d_ff, name=f"{w.name}[d_ff={args.d_ff}]")
    if args.gemm_vs_library:
        run_gemm_vs_library(args, w)
    elif args.route_only:
        run_route_only(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
