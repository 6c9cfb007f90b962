"""Thin ctypes binding of libmoe.so (include/moe.h).

Argument marshalling only: torch tensors become device pointers, the
current torch CUDA stream becomes the call's stream, status codes become
exceptions.  Every step of the layer runs in the library's CUDA kernels.
There is no CPU fallback: a missing library, a CPU tensor or a machine
without CUDA raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

from .inputs import Workload

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK, MOE_ERR_TIMEOUT = 4, 5, 6
MOE_F32, MOE_BF16 = 0, 1
MOE_ACT_RELU, MOE_ACT_SWIGLU = 0, 1
MOE_TOKEN_CHOICE, MOE_EXPERT_CHOICE = 0, 1
MOE_ROUTE_SOFTMAX, MOE_ROUTE_BIAS, MOE_ROUTE_LOAD = 0, 1, 2
ROUTE_RULES = {"softmax": MOE_ROUTE_SOFTMAX, "bias": MOE_ROUTE_BIAS, "load": MOE_ROUTE_LOAD}

EXPORTS = ("moe_query_sizes", "moe_route", "moe_gate", "moe_permute", "moe_expert_ffn",
           "moe_combine", "moe_forward", "moe_check_device_errors", "moe_workspace_init",
           "moe_status_string", "moe_permute_noalloc", "moe_forward_timed",
           "moe_route_bias_update", "moe_query_backward_size", "moe_backward",
           "moe_kernel_launches", "moe_workspace_set_wait_limit", "moe_forward_host")


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int32), ("E", ctypes.c_int32),
                ("S", ctypes.c_int32), ("k", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("keep_num", ctypes.c_int32),
                ("keep_den", ctypes.c_int32), ("ec_capacity", ctypes.c_int32),
                ("n_groups", ctypes.c_int32), ("topk_groups", ctypes.c_int32),
                ("renormalize", ctypes.c_int32), ("act", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("route_rule", ctypes.c_int32), ("route_alpha", ctypes.c_float),
                ("local_groups", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class MoeSizes(ctypes.Structure):
    _fields_ = [("rows_cap", ctypes.c_int64), ("rows_total", ctypes.c_int64),
                ("tok_rows_len", ctypes.c_int64), ("step_workspace", ctypes.c_size_t),
                ("workspace", ctypes.c_size_t), ("capacity", ctypes.c_int64),
                ("permute_workspace", ctypes.c_size_t), ("host_workspace", ctypes.c_size_t)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_layer_63_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, cfgp = ctypes.c_void_p, ctypes.POINTER(MoeConfig)
        sz = ctypes.c_size_t
        sig = {
            "moe_query_sizes": [cfgp, ctypes.POINTER(MoeSizes)],
            "moe_route": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_gate": [cfgp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_route_bias_update": [cfgp, vp, vp, ctypes.c_float, vp],
            "moe_query_backward_size": [cfgp, ctypes.POINTER(ctypes.c_size_t)],
            "moe_backward": [cfgp] + [vp] * 14 + [vp, sz, vp, sz, vp],
            "moe_permute": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_expert_ffn": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_combine": [cfgp, vp, vp, vp, vp],
            "moe_forward": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "moe_forward_timed": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                  ctypes.POINTER(ctypes.c_void_p), vp],
            "moe_forward_host": [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp, vp],
            "moe_check_device_errors": [vp, sz, vp, ctypes.POINTER(ctypes.c_uint32)],
            "moe_workspace_init": [vp, sz, vp],
            "moe_workspace_set_wait_limit": [vp, sz, ctypes.c_uint64, vp],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_kernel_launches.argtypes = []
        L.moe_kernel_launches.restype = ctypes.c_uint64
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def kernel_launches() -> int:
    """Kernels the library has launched since it was loaded (host counter)."""
    return int(lib().moe_kernel_launches())


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoeError(fn, status)


def _ptr(t: torch.Tensor | None, numel: int | None = None, dtype: torch.dtype | None = None):
    """Device pointer of a contiguous CUDA tensor on the current device; with
    numel / dtype given, also checks that it holds at least numel elements of
    that dtype (a short buffer would be written past its end)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmoe takes CUDA tensors only (no CPU path)")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"expected {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"buffer of {t.numel()} elements, {numel} needed")
    return t.data_ptr()


def _stream(stream: torch.cuda.Stream | None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ws(ws: torch.Tensor):
    return _ptr(ws), ws.numel() * ws.element_size()


# ---------------------------------------------------------------------------
# configuration
# ---------------------------------------------------------------------------

def config_from_workload(w: Workload, T: int | None = None) -> MoeConfig:
    T = w.T if T is None else T
    c = MoeConfig()
    c.T, c.d_model, c.E, c.S, c.k, c.d_ff = T, w.d_model, w.E, w.S, w.k, w.d_ff
    # the library derives the expert capacity from the factor (per local group)
    c.capacity_factor = w.capacity_factor if w.mode == "tc" else 0.0
    c.keep_num, c.keep_den = w.keep_num, w.keep_den
    if T != w.T:
        w = w.with_tokens(T)
    c.ec_capacity = w.ec_capacity if w.mode == "ec" else 0
    c.n_groups, c.topk_groups = w.n_groups, w.topk_groups
    c.renormalize = int(w.renormalize)
    c.act = MOE_ACT_SWIGLU if w.act == "swiglu" else MOE_ACT_RELU
    c.mode = MOE_EXPERT_CHOICE if w.mode == "ec" else MOE_TOKEN_CHOICE
    c.dtype = MOE_F32 if w.dtype == "f32" else MOE_BF16
    c.route_rule = ROUTE_RULES[w.route_rule]
    c.route_alpha = w.route_alpha
    c.local_groups = w.local_groups
    return c


@dataclass
class Sizes:
    rows_cap: int
    rows_total: int
    tok_rows_len: int
    step_workspace: int
    workspace: int
    capacity: int
    permute_workspace: int
    host_workspace: int


_sizes_cache: dict[bytes, Sizes] = {}


def query_sizes(cfg: MoeConfig) -> Sizes:
    key = bytes(cfg)
    hit = _sizes_cache.get(key)
    if hit is not None:
        return hit
    out = MoeSizes()
    _check("moe_query_sizes", lib().moe_query_sizes(ctypes.byref(cfg), ctypes.byref(out)))
    s = Sizes(out.rows_cap, out.rows_total, out.tok_rows_len, out.step_workspace, out.workspace,
              out.capacity, out.permute_workspace, out.host_workspace)
    if len(_sizes_cache) < 256:
        _sizes_cache[key] = s
    return s


class _Need:
    """Element counts and dtypes of a configuration's buffers, for the size
    checks of the bindings (a short output buffer would be written past its
    end by the kernels)."""

    def __init__(self, cfg: MoeConfig):
        s = query_sizes(cfg)
        self.dt = torch.float32 if cfg.dtype == MOE_F32 else torch.bfloat16
        T, E, d, f = cfg.T, cfg.E, cfg.d_model, cfg.d_ff
        k = cfg.k if cfg.mode == MOE_TOKEN_CHOICE else 0
        self.td, self.te, self.tk, self.e = T * d, T * E, T * k, E
        self.rows_cap, self.tok_rows = max(s.rows_cap, 1), s.tok_rows_len
        self.x_perm = max(s.rows_cap, 1) * d
        self.h, self.y_rows = s.rows_total * f, s.rows_total * d


def new_workspace(cfg: MoeConfig, device="cuda", step_only: bool = False,
                  host: bool = False) -> torch.Tensor:
    """A zeroed workspace tensor (uint8) of the size the configuration needs
    (step entry points, moe_forward, or moe_forward_host)."""
    s = query_sizes(cfg)
    n = s.step_workspace if step_only else (s.host_workspace if host else s.workspace)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def moe_route(cfg, x, w_router, bias, logits, probs, topk_idx, topk_gate, ws, stream=None, *,
              route_state=None):
    wp, wn = _ws(ws)
    n = _Need(cfg)
    _check("moe_route", lib().moe_route(ctypes.byref(cfg), _ptr(x, n.td, n.dt), _ptr(w_router),
                                        _ptr(bias), _ptr(route_state), _ptr(logits, n.te, torch.float32),
                                        _ptr(probs, n.te, torch.float32),
                                        _ptr(topk_idx, n.tk, torch.int32),
                                        _ptr(topk_gate, n.tk, torch.float32), wp, wn, _stream(stream)))


def moe_gate(cfg, logits, probs, topk_idx, topk_gate, ws, stream=None, *, route_state=None):
    wp, wn = _ws(ws)
    n = _Need(cfg)
    _check("moe_gate", lib().moe_gate(ctypes.byref(cfg), _ptr(logits, n.te, torch.float32),
                                      _ptr(route_state), _ptr(probs, n.te, torch.float32),
                                      _ptr(topk_idx, n.tk, torch.int32),
                                      _ptr(topk_gate, n.tk, torch.float32), wp, wn, _stream(stream)))


def moe_route_bias_update(cfg, counts, route_bias, gamma: float, stream=None):
    """DeepSeek-V3's bias step: route_bias[e] -/+ gamma for experts above /
    below the mean load T*k/E, in place."""
    _check("moe_route_bias_update", lib().moe_route_bias_update(
        ctypes.byref(cfg), _ptr(counts), _ptr(route_bias), float(gamma), _stream(stream)))


def moe_permute(cfg, x, topk_idx, topk_gate, probs, counts, offsets, tok_rows, row_token, row_gate,
                x_perm, n_dropped, ws, stream=None):
    wp, wn = _ws(ws)
    n = _Need(cfg)
    _check("moe_permute", lib().moe_permute(
        ctypes.byref(cfg), _ptr(x, n.td, n.dt), _ptr(topk_idx), _ptr(topk_gate), _ptr(probs),
        *_permute_outputs(n, counts, offsets, tok_rows, row_token, row_gate, x_perm, n_dropped),
        wp, wn, _stream(stream)))


def _permute_outputs(n: _Need, counts, offsets, tok_rows, row_token, row_gate, x_perm, n_dropped):
    i32 = torch.int32
    return (_ptr(counts, n.e, i32), _ptr(offsets, n.e + 1, i32), _ptr(tok_rows, n.tok_rows, i32),
            _ptr(row_token, n.rows_cap, i32), _ptr(row_gate, n.rows_cap, torch.float32),
            _ptr(x_perm, n.x_perm, n.dt), _ptr(n_dropped, 1, i32))


def moe_expert_ffn(cfg, x, x_perm, offsets, row_gate, w1, w3, w2, h, y_rows, ws, stream=None):
    wp, wn = _ws(ws)
    n = _Need(cfg)
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        ctypes.byref(cfg), _ptr(x, n.td, n.dt), _ptr(x_perm, None, n.dt), _ptr(offsets), _ptr(row_gate),
        _ptr(w1, None, n.dt), _ptr(w3, None, n.dt), _ptr(w2, None, n.dt), _ptr(h, n.h, n.dt),
        _ptr(y_rows, n.y_rows, n.dt), wp, wn, _stream(stream)))


def moe_combine(cfg, y_rows, tok_rows, y, stream=None):
    n = _Need(cfg)
    _check("moe_combine", lib().moe_combine(ctypes.byref(cfg), _ptr(y_rows, n.y_rows, n.dt),
                                            _ptr(tok_rows, n.tok_rows, torch.int32),
                                            _ptr(y, n.td, n.dt), _stream(stream)))


def moe_forward(cfg, x, w_router, bias, w1, w3, w2, y, counts_out, ws, stream=None, *,
                route_state=None):
    wp, wn = _ws(ws)
    n = _Need(cfg)
    _check("moe_forward", lib().moe_forward(
        ctypes.byref(cfg), _ptr(x, n.td, n.dt), _ptr(w_router), _ptr(bias), _ptr(route_state),
        _ptr(w1, None, n.dt), _ptr(w3, None, n.dt), _ptr(w2, None, n.dt), _ptr(y, n.td, n.dt),
        _ptr(counts_out, n.e, torch.int32), wp, wn, _stream(stream)))


def _host_ptr(t: torch.Tensor, numel: int, dtype: torch.dtype):
    """Address of a contiguous host (CPU) tensor of at least numel elements."""
    if t.is_cuda:
        raise ValueError("moe_forward_host takes host (CPU) tensors for x and y")
    if not t.is_contiguous() or t.dtype != dtype or t.numel() < numel:
        raise ValueError(f"expected a contiguous {dtype} host tensor of {numel} elements")
    return t.data_ptr()


def moe_forward_host(cfg, x_host, w_router, bias, w1, w3, w2, y_host, counts_out, ws, stream=None,
                     copy_in=None, copy_out=None, *, route_state=None):
    """moe_forward on host buffers: x_host is copied in, y comes back to
    y_host, queued on the streams without a host sync (page-locked tensors
    make the copies asynchronous).  copy_in / copy_out: streams for the two
    copies (None: `stream`)."""
    wp, wn = _ws(ws)
    dt = torch.float32 if cfg.dtype == MOE_F32 else torch.bfloat16
    n = cfg.T * cfg.d_model
    cin = None if copy_in is None else copy_in.cuda_stream
    cout = None if copy_out is None else copy_out.cuda_stream
    _check("moe_forward_host", lib().moe_forward_host(
        ctypes.byref(cfg), _host_ptr(x_host, n, dt), _ptr(w_router), _ptr(bias), _ptr(route_state),
        _ptr(w1), _ptr(w3), _ptr(w2), _host_ptr(y_host, n, dt), _ptr(counts_out), wp, wn,
        _stream(stream), cin, cout))


def moe_forward_timed(cfg, x, w_router, bias, w1, w3, w2, y, counts_out, ws, events, stream=None, *,
                      route_state=None):
    """moe_forward recording 5 torch CUDA events at its phase boundaries
    (before routing, after routing, after permutation, after the expert FFNs,
    after the combine).  Each event must have been recorded once before, so
    that its CUDA handle exists."""
    wp, wn = _ws(ws)
    handles = (ctypes.c_void_p * 5)(*[ev.cuda_event if ev is not None else None for ev in events])
    n = _Need(cfg)
    _check("moe_forward_timed", lib().moe_forward_timed(
        ctypes.byref(cfg), _ptr(x, n.td, n.dt), _ptr(w_router), _ptr(bias), _ptr(route_state),
        _ptr(w1, None, n.dt), _ptr(w3, None, n.dt), _ptr(w2, None, n.dt), _ptr(y, n.td, n.dt),
        _ptr(counts_out, n.e, torch.int32), wp, wn, handles, _stream(stream)))


def query_backward_size(cfg: MoeConfig) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_query_backward_size", lib().moe_query_backward_size(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def moe_backward(cfg, x, w_router, bias, w1, w3, w2, dy, dx, dw_router, dbias, dw1, dw3, dw2, ws, bws,
                 stream=None, *, route_state=None):
    """Gradients of sum(dy * y) for the forward that last ran on ws (routing fixed)."""
    wp, wn = _ws(ws)
    bp, bn = _ws(bws)
    _check("moe_backward", lib().moe_backward(
        ctypes.byref(cfg), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(route_state), _ptr(w1), _ptr(w3),
        _ptr(w2), _ptr(dy), _ptr(dx), _ptr(dw_router), _ptr(dbias), _ptr(dw1), _ptr(dw3), _ptr(dw2),
        wp, wn, bp, bn, _stream(stream)))


def moe_check_device_errors(ws, stream=None) -> int:
    """Blocks on the stream; returns the raw error bits and raises if any is set."""
    wp, wn = _ws(ws)
    flags = ctypes.c_uint32(0)
    st = lib().moe_check_device_errors(wp, wn, _stream(stream), ctypes.byref(flags))
    _check("moe_check_device_errors", st)
    return flags.value


def moe_workspace_init(ws, stream=None):
    wp, wn = _ws(ws)
    _check("moe_workspace_init", lib().moe_workspace_init(wp, wn, _stream(stream)))


def moe_workspace_set_wait_limit(ws, limit_ns: int, stream=None):
    """Time limit of the device-side waits of launches on ws (0: default 2 s)."""
    wp, wn = _ws(ws)
    _check("moe_workspace_set_wait_limit",
           lib().moe_workspace_set_wait_limit(wp, wn, int(limit_ns), _stream(stream)))


# ---------------------------------------------------------------------------
# convenience: buffers of the step API, and a layer object
# ---------------------------------------------------------------------------

@dataclass
class StepBuffers:
    logits: torch.Tensor
    probs: torch.Tensor
    topk_idx: torch.Tensor | None
    topk_gate: torch.Tensor | None
    counts: torch.Tensor
    offsets: torch.Tensor
    tok_rows: torch.Tensor
    row_token: torch.Tensor
    row_gate: torch.Tensor
    x_perm: torch.Tensor
    n_dropped: torch.Tensor
    h: torch.Tensor
    y_rows: torch.Tensor
    y: torch.Tensor
    ws: torch.Tensor


def step_buffers(cfg: MoeConfig, device="cuda") -> StepBuffers:
    s = query_sizes(cfg)
    dt = torch.float32 if cfg.dtype == MOE_F32 else torch.bfloat16
    T, E, d, f = cfg.T, cfg.E, cfg.d_model, cfg.d_ff
    tc = cfg.mode == MOE_TOKEN_CHOICE
    i32, f32 = torch.int32, torch.float32
    return StepBuffers(
        logits=torch.empty(T, E, dtype=f32, device=device),
        probs=torch.empty(T, E, dtype=f32, device=device),
        topk_idx=torch.empty(T, cfg.k, dtype=i32, device=device) if tc else None,
        topk_gate=torch.empty(T, cfg.k, dtype=f32, device=device) if tc else None,
        counts=torch.empty(E, dtype=i32, device=device),
        offsets=torch.empty(E + 1, dtype=i32, device=device),
        tok_rows=torch.empty(s.tok_rows_len, dtype=i32, device=device),
        row_token=torch.empty(max(s.rows_cap, 1), dtype=i32, device=device),
        row_gate=torch.empty(max(s.rows_cap, 1), dtype=f32, device=device),
        x_perm=torch.empty(max(s.rows_cap, 1), d, dtype=dt, device=device),
        n_dropped=torch.empty(1, dtype=i32, device=device),
        h=torch.empty(s.rows_total, f, dtype=dt, device=device),
        y_rows=torch.empty(s.rows_total, d, dtype=dt, device=device),
        y=torch.empty(T, d, dtype=dt, device=device),
        ws=new_workspace(cfg, device, step_only=True),
    )


class MoELayer:
    """The layer's weights plus a workspace; ``layer(x)`` runs moe_forward."""

    def __init__(self, cfg: MoeConfig, w_router, w1, w2, w3=None, bias=None, route_state=None):
        self.cfg = cfg
        self.w_router, self.w1, self.w2, self.w3, self.bias = w_router, w1, w2, w3, bias
        if route_state is None and cfg.route_rule != MOE_ROUTE_SOFTMAX:
            route_state = torch.zeros(cfg.E, dtype=torch.float32, device=w1.device)
        self.route_state = route_state     # routing bias (DeepSeek-V3) or utilisation
        self.ws = new_workspace(cfg, w1.device)
        self.counts = torch.empty(cfg.E, dtype=torch.int32, device=w1.device)

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        y = out if out is not None else torch.empty_like(x)
        moe_forward(self.cfg, x, self.w_router, self.bias, self.w1, self.w3, self.w2, y,
                    self.counts, self.ws, stream, route_state=self.route_state)
        return y

    def backward(self, x: torch.Tensor, dy: torch.Tensor, stream=None) -> dict:
        """Gradients of sum(dy * y) for the last ``self(x)`` (same x), routing
        fixed: dx, dw_router, dbias (when the layer has a logit bias), dw1,
        dw3 (SwiGLU), dw2, all fp32."""
        if getattr(self, "bws", None) is None:
            self.bws = torch.empty(max(query_backward_size(self.cfg), 256), dtype=torch.uint8,
                                   device=x.device)
        f32 = dict(dtype=torch.float32, device=x.device)
        g = {"dx": torch.empty(x.shape, **f32), "dw_router": torch.empty(self.w_router.shape, **f32),
             "dbias": torch.empty(self.bias.shape, **f32) if self.bias is not None else None,
             "dw1": torch.empty(self.w1.shape, **f32),
             "dw3": torch.empty(self.w3.shape, **f32) if self.w3 is not None else None,
             "dw2": torch.empty(self.w2.shape, **f32)}
        moe_backward(self.cfg, x, self.w_router, self.bias, self.w1, self.w3, self.w2, dy, g["dx"],
                     g["dw_router"], g["dbias"], g["dw1"], g["dw3"], g["dw2"], self.ws, self.bws,
                     stream, route_state=self.route_state)
        return g

    def update_route_bias(self, gamma: float, stream=None):
        """DeepSeek-V3's bias step from the last forward's counts."""
        moe_route_bias_update(self.cfg, self.counts, self.route_state, gamma, stream)


class HostPipeline:
    """Serving from host memory through moe_forward_host: batches of T tokens
    in page-locked host buffers go through ``layer`` and their outputs come
    back to page-locked host buffers.  Two workspaces are used in turn and
    the copies run on their own streams, so the host-to-device copy of a
    batch and the device-to-host copy of the one before it overlap the
    forward in between; the forwards stay in order on one stream (the library
    orders the calls that share a workspace).

        pipe = HostPipeline(layer)
        for x_h, y_h in batches:          # pinned [T, d] tensors
            pipe.submit(x_h, y_h)
        pipe.synchronize()                # every y_h is now filled
    """

    def __init__(self, layer: MoELayer, before_forward=None):
        self.layer = layer
        dev = layer.w1.device
        self.ws = [new_workspace(layer.cfg, dev, host=True) for _ in range(2)]
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_comp = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.before_forward = before_forward     # optional callable, run on the compute stream
        self.i = 0

    def submit(self, x_host: torch.Tensor, y_host: torch.Tensor) -> None:
        """Queue one batch (the host tensors must stay untouched until synchronize)."""
        L = self.layer
        if self.before_forward is not None:
            with torch.cuda.stream(self.s_comp):
                self.before_forward()
        moe_forward_host(L.cfg, x_host, L.w_router, L.bias, L.w1, L.w3, L.w2, y_host, L.counts,
                         self.ws[self.i & 1], self.s_comp, self.s_in, self.s_out,
                         route_state=L.route_state)
        self.i += 1

    def synchronize(self):
        for st in (self.s_in, self.s_comp, self.s_out):
            st.synchronize()


# ---------------------------------------------------------------------------
# moe_permute without a workspace (callers that cannot allocate device memory)
# ---------------------------------------------------------------------------

NOALLOC_SCRATCH_BYTES = 8 << 20
_noalloc_fn = None


def _noalloc():
    """moe_permute_noalloc with its C signature declared (once)."""
    global _noalloc_fn
    if _noalloc_fn is None:
        f = lib().moe_permute_noalloc
        f.argtypes = [ctypes.POINTER(MoeConfig)] + [ctypes.c_void_p] * 12
        f.restype = ctypes.c_int
        _noalloc_fn = f
    return _noalloc_fn


def moe_permute_noalloc(cfg, x, topk_idx, topk_gate, probs, counts, offsets, tok_rows, row_token,
                        row_gate, x_perm, n_dropped, stream=None):
    """moe_permute with its scratch in the library's fixed 8 MiB device array.

    For callers that cannot allocate device memory (a plugin handed only its
    inputs and outputs, or a process with a fixed footprint after start-up).
    The first call on a device looks up the array's address: make it before
    any stream capture.  Calls that overlap on the GPU race on the array.
    """
    n = _Need(cfg)
    _check("moe_permute_noalloc", _noalloc()(
        ctypes.byref(cfg), _ptr(x, n.td, n.dt), _ptr(topk_idx), _ptr(topk_gate), _ptr(probs),
        *_permute_outputs(n, counts, offsets, tok_rows, row_token, row_gate, x_perm, n_dropped),
        _stream(stream)))
