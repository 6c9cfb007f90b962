"""CPU oracle for the forward pass of a sparse Mixture-of-Experts FFN layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / reference leg of ``bench.py`` may import this module.
It shares no code with the CUDA path and imports nothing from it; it takes
plain numpy arrays (bf16 tensors arrive as their raw uint16 bit patterns, or
as float32/float64 arrays holding the exact widened values).

What it computes, step by step, and the passage each step follows:

1. Router logits ``l = x . W_r^T (+ b)``: the router is "an FFN plus a
   softmax layer" ("大语言模型并行策略（七）：专家并行", section
   "Mixture of Experts (MoE)"); read here as one bias-free linear layer over
   the routed experts.  Accumulated in float64, rounded once to fp32.
2. Softmax gating ``p_i = exp(g_i) / sum_j exp(g_j)`` ("MoE技术演进",
   "Adaptive Mixtures of Local Experts", gating-network equation).  Exact
   mathematics, but evaluated by a fixed fp32 recipe (``exp_det`` and a
   sequential ascending-expert sum) because expert-choice selection and
   affinity-based token dropping compare probabilities across tokens: both
   sides must take those integer decisions in the same precision.
3. Selection:
   a. token choice top-k by weight, lower expert index on ties ("MoE技术演进",
      "Adaptive Mixtures of Local Experts", selector; GShard section 1 top-2);
      optional group-limited routing (DeepSeek-V2 section 3, device-limited
      routing: pick M groups, then top-K inside them);
   b. expert capacity with overflow dropped to the residual (GShard
      section 1, expert capacity C = O(N/E));
   c. per-expert affinity-based token dropping, keep the top fraction
      (DeepSeek-V2 section 5, token-dropping strategy);
   d. expert choice: each expert takes its top-C tokens (LocMoE+ article,
      token-choice vs expert-choice routers);
   e. shared experts applied to every token with gate 1 (DeepSeekMoE
      section 2, shared expert isolation equation);
   f. selection-key variants: DeepSeek-V3's auxiliary-loss-free balancing
      (select on s + b, gate s + b; "MoE技术演进", DeepSeek-V3 item 1) with
      its per-step bias update, and load-aware top-k (select on
      g + alpha (1 - u); "MoE技术演进", interview question Q3, item 3);
   g. GShard local group dispatching: the batch cut into G groups that
      dispatch independently, capacity per group ("MoE技术演进", GShard
      item 1).
4. Permutation into expert-contiguous rows (the single-GPU counterpart of the
   count-then-fill send buffers, "大语言模型并行策略（七）：专家并行",
   section "MoE 中的 all-to-all 通信").
5. Expert FFNs ``w_o . ReLU(w_i . x)`` (GShard section 3, FFN_e equation) or
   SwiGLU with 3 * d_model * d_moe parameters ("大语言模型并行策略（七）",
   parameter-count notes), and the gate-weighted combine
   ``y_s = sum_e G_{s,e} FFN_e(x_s)`` (GShard section 3) plus the shared
   experts' sum (DeepSeekMoE section 2).  Float64 throughout; the residual
   ``+ u`` of the DeepSeekMoE equations is left to the caller.

Readings where the pages are silent (each is repeated in the design notes):
capacity ``C = ceil(cf * k * T / E)`` with one group; drop priority
``q = j * T + t`` (every first choice before any second choice, lower token
first); top-k keys are the fp32 logits; gates are the unnormalised
probabilities unless ``renormalize``; group score = max logit in a
contiguous group; keep-fraction keys = p, ties to the lower token, applied
per expert after top-k; expert-choice keys = p, ties to the lower token,
segment order ascending token; SwiGLU = ``W_down (SiLU(W_gate x) * W_up x)``.

Every function here is pinned by tests under ``tests/`` against closed forms,
brute-force enumeration, special cases that reduce to a dense FFN or a dense
soft mixture, and invariants; none is "parity unpinned".
"""
from __future__ import annotations

import math
from fractions import Fraction
from dataclasses import dataclass

import numpy as np

F32 = np.float32

# --------------------------------------------------------------------------
# input decoding
# --------------------------------------------------------------------------


def widen(a: np.ndarray) -> np.ndarray:
    """Exact float64 values of an input array.

    uint16 arrays are bf16 bit patterns (the upper half of an fp32 word);
    float arrays are taken as they are.
    """
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------------
# step 2 arithmetic: a fixed fp32 exponential
# --------------------------------------------------------------------------

# Cody-Waite range reduction: ln 2 split into a 16-bit head (so n * LN2_HI is
# exact for |n| < 256) and the fp32-rounded remainder.
LOG2E = F32(1.4426950408889634)
LN2_HI = F32(45426.0 / 65536.0)                       # 0.693145751953125
LN2_LO = F32(math.log(2.0) - 45426.0 / 65536.0)       # 1.4286068e-06
# Taylor coefficients 1/i!, i = 0..7, rounded to fp32
EXP_COEF = tuple(F32(1.0 / math.factorial(i)) for i in range(8))
EXP_FLUSH = F32(-87.0)     # below this exp(z) < 2**-125: returned as 0


def exp_det(z: np.ndarray) -> np.ndarray:
    """exp(z) for fp32 z <= 0, by one fixed sequence of rounded fp32 ops.

    n = rint(z * log2 e); r = (z - n ln2_hi) - n ln2_lo; a degree-7 Taylor
    polynomial of e^r in Horner form, each step one rounded multiply and one
    rounded add (no fused multiply-add); then the exact scale by 2**n built
    from exponent bits.  z < -87 returns 0.  Error against exp: a few ulp
    (pinned in the tests).
    """
    z = np.asarray(z, dtype=F32)
    with np.errstate(over="ignore", invalid="ignore"):      # flushed lanes may overflow
        return _exp_det(z)


def _exp_det(z: np.ndarray) -> np.ndarray:
    n = np.rint(z * LOG2E).astype(F32)
    r = (z - n * LN2_HI).astype(F32)
    r = (r - n * LN2_LO).astype(F32)
    p = np.full_like(z, EXP_COEF[7])
    for c in EXP_COEF[6::-1]:
        p = (p * r).astype(F32)
        p = (p + c).astype(F32)
    ni = np.clip(n, -126, 0).astype(np.int32)
    scale = ((ni + 127).astype(np.uint32) << np.uint32(23)).view(F32)
    out = (p * scale).astype(F32)
    return np.where(z < EXP_FLUSH, F32(0.0), out).astype(F32)


# --------------------------------------------------------------------------
# steps 1-2
# --------------------------------------------------------------------------


def router_logits(x: np.ndarray, w_router: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """l[t, e] = sum_i x[t, i] W_r[e, i] (+ b[e]) in float64, rounded to fp32."""
    acc = widen(x) @ widen(w_router).T
    if bias is not None:
        acc = acc + widen(bias)[None, :]
    return acc.astype(F32)


def softmax_det(logits: np.ndarray) -> np.ndarray:
    """p[t, e] = exp(l - m) / sum_e' exp(l' - m), m = max_e l, in fixed fp32.

    z = l - m is one rounded fp32 subtraction; exp is ``exp_det``; the
    denominator is summed sequentially in ascending expert order in fp32;
    the quotient is one rounded fp32 division.
    """
    l = np.asarray(logits, dtype=F32)
    m = l.max(axis=1, keepdims=True)
    z = (l - m).astype(F32)
    e = exp_det(z)
    s = e[:, 0].copy()
    for j in range(1, l.shape[1]):
        s = (s + e[:, j]).astype(F32)
    return (e / s[:, None]).astype(F32)


# --------------------------------------------------------------------------
# step 3a: token-choice top-k
# --------------------------------------------------------------------------


def group_limited_mask(logits: np.ndarray, n_groups: int, topk_groups: int) -> np.ndarray:
    """Boolean [T, E]: experts inside each token's top ``topk_groups`` groups.

    Groups are ``n_groups`` contiguous blocks of E / n_groups experts; a
    group's score is its largest logit; groups rank by score, lower group
    index on ties.
    """
    l = np.asarray(logits, dtype=F32)
    T, E = l.shape
    gsz = E // n_groups
    score = l.reshape(T, n_groups, gsz).max(axis=2)
    order = np.argsort(-score, axis=1, kind="stable")       # stable: lower group first on ties
    chosen = np.zeros((T, n_groups), dtype=bool)
    np.put_along_axis(chosen, order[:, :topk_groups], True, axis=1)
    return np.repeat(chosen, gsz, axis=1)


ROUTE_RULES = ("softmax", "bias", "load")


def selection_keys(logits: np.ndarray, probs: np.ndarray, rule: str = "softmax",
                   state: np.ndarray | None = None, alpha: float = 0.0):
    """Per (token, expert): the fp32 key top-k selects on and the gate a
    chosen expert receives.

    "softmax": key = the logit g, gate = p (the plain selector).
    "bias"   : DeepSeek-V3's auxiliary-loss-free balancing ("MoE技术演进",
               DeepSeek-V3 item 1): key = s + b_e, one rounded fp32 add,
               with the affinity s read as the softmax probability p and
               b = ``state`` the per-expert routing bias; the gate of a chosen
               expert is s + b_e, as the printed formula gives it.
    "load"   : load-aware top-k ("MoE技术演进", interview question Q3,
               item 3): key = g_e + alpha * (1 - u_e) with g the logit and
               u = ``state`` the expert's historical utilisation; in fp32
               o_e = alpha * (1 - u_e) (two rounded operations), key = g + o_e
               (one rounded add); the gate stays p.
    """
    l = np.asarray(logits, dtype=F32)
    p = np.asarray(probs, dtype=F32)
    if rule == "softmax":
        return l, p
    st = np.asarray(state, dtype=F32)
    if rule == "bias":
        key = (p + st[None, :]).astype(F32)
        return key, key
    if rule == "load":
        off = (F32(alpha) * (F32(1.0) - st).astype(F32)).astype(F32)
        return (l + off[None, :]).astype(F32), p
    raise ValueError(rule)


def bias_update(counts: np.ndarray, bias: np.ndarray, T: int, k: int, gamma: float) -> np.ndarray:
    """DeepSeek-V3's per-step update of the routing bias ("MoE技术演进",
    DeepSeek-V3 item 1): an expert with more assignments than the mean T*k/E
    (overloaded) lowers its bias by gamma, one with fewer raises it by gamma,
    one exactly at the mean keeps it.  The load test is exact integer
    arithmetic (c_e * E against T * k); the step is one rounded fp32 add."""
    c = np.asarray(counts, dtype=np.int64)
    b = np.asarray(bias, dtype=F32)
    E = len(c)
    g = F32(gamma)
    over = c * E > T * k
    under = c * E < T * k
    out = b.copy()
    out[over] = (b[over] - g).astype(F32)
    out[under] = (b[under] + g).astype(F32)
    return out


def topk_route(logits: np.ndarray, probs: np.ndarray, k: int, n_groups: int = 0,
               topk_groups: int = 0, renormalize: bool = False, rule: str = "softmax",
               state: np.ndarray | None = None, alpha: float = 0.0):
    """Per token: the k experts with the largest selection keys, in rank order.

    Keys and gates come from ``selection_keys`` (plain: the logits, so by
    monotonicity of softmax the top-k of p with exact ties broken by index).
    A strictly larger key ranks first; equal keys go to the lower expert
    index.  With group limits only experts of the chosen groups compete (a
    group's score is its largest key).  Gate = that of the chosen expert, or
    gate / (sum of the chosen gates, summed in rank order in fp32) when
    ``renormalize``.
    Returns (topk_idx int32 [T, k], topk_gate fp32 [T, k]).
    """
    key, gsrc = selection_keys(logits, probs, rule, state, alpha)
    keys = -key.astype(np.float64)
    if n_groups > 0:
        allowed = group_limited_mask(key, n_groups, topk_groups)
        keys = np.where(allowed, keys, np.inf)
    order = np.argsort(keys, axis=1, kind="stable")           # ties keep ascending expert index
    idx = order[:, :k].astype(np.int32)
    gate = np.take_along_axis(np.asarray(gsrc, dtype=F32), idx, axis=1).astype(F32)
    if renormalize:
        s = gate[:, 0].copy()
        for j in range(1, k):
            s = (s + gate[:, j]).astype(F32)
        gate = (gate / s[:, None]).astype(F32)
    return idx, gate


# --------------------------------------------------------------------------
# steps 3b-3d and 4: dispatch / permutation
# --------------------------------------------------------------------------


@dataclass
class Dispatch:
    """Expert-contiguous row layout produced by selection + permutation.

    counts[e]   assignments made to expert e before any drop (token choice),
                or the tokens it picked (expert choice)
    kept[e]     rows expert e actually processes
    offsets     exclusive scan of kept, length E + 1
    row_token   token of each row, length offsets[E]
    row_gate    gate of each row (fp32)
    tok_rows    token choice: [T, k], the row of (t, j) or -1 when dropped;
                expert choice: [E, T], the row of (e, t) or -1
    n_dropped   token choice: assignments dropped by capacity / keep-fraction
    """

    counts: np.ndarray
    kept: np.ndarray
    offsets: np.ndarray
    row_token: np.ndarray
    row_gate: np.ndarray
    tok_rows: np.ndarray
    n_dropped: int


def capacity_from_factor(T: int, E: int, k: int, capacity_factor: float) -> int:
    """C = ceil(cf * k * T / E); 0 means unlimited (cf <= 0).

    GShard section 1 of "MoE技术演进" fixes only C = O(N/E) (2N/(G*E) per
    group for top-2); the factor form is the workloads'.  The ceiling is taken
    of the exact product for the binary value of cf (a fraction, no rounding
    before the ceiling): a floating-point product could land on either side
    of an integer."""
    if capacity_factor <= 0:
        return 0
    return int(math.ceil(Fraction(capacity_factor) * k * T / E))


def keep_count(n: np.ndarray, keep_num: int, keep_den: int) -> np.ndarray:
    """ceil(n * num / den) in integers; num = den = 0 keeps everything."""
    n = np.asarray(n, dtype=np.int64)
    if keep_den <= 0:
        return n
    return (n * keep_num + keep_den - 1) // keep_den


def _priority_ranks(topk_idx: np.ndarray, E: int, local_groups: int = 1):
    """Stable counting sort of assignments by expert in priority order.

    Assignment (t, j) is numbered q = j * T + t.  With one group its priority
    is q itself.  With G local groups (tokens cut into G contiguous groups of
    T/G) the priority is group-major: group g's assignments in the order
    j * (T/G) + (t - g T/G), then group g + 1's.  Returns the expert of each
    q, the q's grouped by expert (ascending priority inside each expert), the
    start of each expert's group, the rank of each q inside its expert and
    local group, and the local group of each q.
    """
    T, k = topk_idx.shape
    G = max(1, int(local_groups))
    Tg = T // G
    e_of_q = np.asarray(topk_idx, dtype=np.int64).T.reshape(-1)     # q = j*T + t
    q = np.arange(T * k)
    t_of_q, j_of_q = q % T, q // T
    g_of_q = t_of_q // Tg
    prio = g_of_q * (k * Tg) + j_of_q * Tg + (t_of_q - g_of_q * Tg)
    by_expert = np.lexsort((prio, e_of_q))                          # by expert, then priority
    counts = np.bincount(e_of_q, minlength=E).astype(np.int64)
    start = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank = np.empty(T * k, dtype=np.int64)
    # rank inside (expert, group): position in the sorted list minus the
    # position of the first assignment of the same (expert, group)
    se, sg = e_of_q[by_expert], g_of_q[by_expert]
    first = np.ones(T * k, dtype=bool)
    first[1:] = (se[1:] != se[:-1]) | (sg[1:] != sg[:-1])
    run_start = np.maximum.accumulate(np.where(first, np.arange(T * k), 0))
    rank[by_expert] = np.arange(T * k) - run_start
    return e_of_q, by_expert, counts, start, rank, g_of_q


def dispatch_token_choice(topk_idx: np.ndarray, topk_gate: np.ndarray, probs: np.ndarray | None,
                          E: int, capacity: int = 0, keep_num: int = 0, keep_den: int = 0,
                          local_groups: int = 1) -> Dispatch:
    """Token-choice dispatch with an optional capacity or keep-fraction.

    Capacity C > 0: the assignment of priority q is kept iff fewer than C
    assignments of smaller q went to the same expert; the rest overflow to
    the residual and contribute nothing here.
    Local groups G > 1 (GShard item 1, "MoE技术演进"): the tokens form G
    contiguous groups of T/G that dispatch independently; C is then the
    capacity of one expert in one group, and ranks count only the group's
    own assignments (T must be a multiple of G; capacity mode only).
    Keep-fraction num/den: expert e keeps ceil(n_e * num / den) of its n_e
    assignments, those with the largest p[t, e] (lower t on ties).
    Rows of an expert are its kept assignments in priority order (group by
    group when G > 1).
    """
    topk_idx = np.asarray(topk_idx)
    T, k = topk_idx.shape
    if local_groups > 1 and (T % local_groups or capacity <= 0):
        raise ValueError("local groups need T % G == 0 and a capacity")
    e_of_q, by_expert, counts, start, rank, _ = _priority_ranks(topk_idx, E, local_groups)
    t_of_q = np.arange(T * k) % T
    keep = np.ones(T * k, dtype=bool)
    if capacity > 0:
        keep = rank < capacity
    elif keep_den > 0:
        p = np.asarray(probs, dtype=F32)
        m = keep_count(counts, keep_num, keep_den)
        for e in range(E):
            qs = by_expert[start[e]:start[e] + counts[e]]
            pe = p[t_of_q[qs], e]
            # sort by p descending, then t ascending
            order = np.lexsort((t_of_q[qs], -pe.astype(np.float64)))
            dropped = qs[order[m[e]:]]
            keep[dropped] = False
    kept = np.bincount(e_of_q[keep], minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(kept)]).astype(np.int64)
    # position among the kept rows of the same expert, in priority order
    kept_rank = np.zeros(T * k, dtype=np.int64)
    for e in range(E):
        qs = by_expert[start[e]:start[e] + counts[e]]
        qk = qs[keep[qs]]
        kept_rank[qk] = np.arange(len(qk))
    slot_q = np.where(keep, offsets[e_of_q] + kept_rank, -1)
    tok_rows = slot_q.reshape(k, T).T.astype(np.int32).copy()
    R = int(offsets[E])
    row_token = np.empty(R, dtype=np.int32)
    row_gate = np.empty(R, dtype=F32)
    gate_q = np.asarray(topk_gate, dtype=F32).T.reshape(-1)
    row_token[slot_q[keep]] = t_of_q[keep]
    row_gate[slot_q[keep]] = gate_q[keep]
    return Dispatch(counts.astype(np.int32), kept.astype(np.int32), offsets.astype(np.int32),
                    row_token, row_gate, tok_rows, int(T * k - keep.sum()))


def dispatch_expert_choice(probs: np.ndarray, C: int) -> Dispatch:
    """Expert choice: expert e takes the C tokens with the largest p[t, e].

    Ties go to the lower token index; rows of an expert are its tokens in
    ascending token order; gate = p[t, e].  A token may be taken by any
    number of experts, including none.
    """
    p = np.asarray(probs, dtype=F32)
    T, E = p.shape
    tok_rows = np.full((E, T), -1, dtype=np.int32)
    row_token = np.empty(E * C, dtype=np.int32)
    row_gate = np.empty(E * C, dtype=F32)
    t = np.arange(T)
    for e in range(E):
        order = np.lexsort((t, -p[:, e].astype(np.float64)))
        chosen = np.sort(order[:C])
        rows = e * C + np.arange(C)
        row_token[rows] = chosen
        row_gate[rows] = p[chosen, e]
        tok_rows[e, chosen] = rows
    counts = np.full(E, C, dtype=np.int32)
    offsets = (np.arange(E + 1) * C).astype(np.int32)
    return Dispatch(counts, counts.copy(), offsets, row_token, row_gate, tok_rows, 0)


def permute_rows(x: np.ndarray, d: Dispatch) -> np.ndarray:
    """x_perm[r] = x[row_token[r]] (bit patterns copied as they are)."""
    return np.asarray(x)[d.row_token]


# --------------------------------------------------------------------------
# step 5: expert FFNs and combine
# --------------------------------------------------------------------------


def expert_ffn(xrows: np.ndarray, w1_e, w2_e, w3_e=None, act: str = "relu") -> np.ndarray:
    """FFN_e of a batch of rows in float64.

    ReLU:   w2 . ReLU(w1 . x)                      (GShard section 3)
    SwiGLU: w2 . (SiLU(w1 . x) * (w3 . x)),  SiLU(z) = z / (1 + e^-z)
    Weight layout: w1, w3 [f, d]; w2 [d, f] (each output neuron's weights
    contiguous along the input dimension).
    """
    xr = widen(xrows)
    g = xr @ widen(w1_e).T
    if act == "relu":
        h = np.maximum(g, 0.0)
    elif act == "swiglu":
        u = xr @ widen(w3_e).T
        h = g / (1.0 + np.exp(-g)) * u
    else:
        raise ValueError(act)
    return h @ widen(w2_e).T


@dataclass
class OracleConfig:
    """The layer's options, as the oracle sees them."""

    E: int
    S: int
    k: int
    act: str = "relu"
    mode: str = "tc"
    capacity: int = 0
    keep_num: int = 0
    keep_den: int = 0
    ec_capacity: int = 0
    n_groups: int = 0
    topk_groups: int = 0
    renormalize: bool = False
    rule: str = "softmax"            # selection keys: "softmax", "bias", "load"
    alpha: float = 0.0               # load-aware coefficient
    local_groups: int = 1            # GShard local groups (capacity mode)


@dataclass
class OracleResult:
    logits: np.ndarray
    probs: np.ndarray
    topk_idx: np.ndarray | None
    topk_gate: np.ndarray | None
    dispatch: Dispatch
    tokens: np.ndarray          # tokens whose output was computed
    y: np.ndarray               # float64 [len(tokens), d]


def route(cfg: OracleConfig, logits: np.ndarray, state: np.ndarray | None = None):
    """Steps 2-4 from given fp32 logits: probabilities, selection, dispatch.
    ``state`` is the per-expert routing bias (rule "bias") or utilisation
    (rule "load")."""
    probs = softmax_det(logits)
    if cfg.mode == "ec":
        return probs, None, None, dispatch_expert_choice(probs, cfg.ec_capacity)
    idx, gate = topk_route(logits, probs, cfg.k, cfg.n_groups, cfg.topk_groups, cfg.renormalize,
                           cfg.rule, state, cfg.alpha)
    disp = dispatch_token_choice(idx, gate, probs, cfg.E, cfg.capacity, cfg.keep_num, cfg.keep_den,
                                 cfg.local_groups)
    return probs, idx, gate, disp


def combine_tokens(cfg: OracleConfig, x, w1, w2, w3, disp: Dispatch, tokens) -> np.ndarray:
    """y_t = sum over t's kept (expert, gate) of gate * FFN_e(x_t) + sum_s FFN_s(x_t).

    Computed per expert on the requested tokens only, in float64.  The
    routed terms are added in the token's k-rank order (expert choice:
    ascending expert), then the shared experts in index order.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    x = np.asarray(x)
    d = x.shape[1]
    y = np.zeros((len(tokens), d), dtype=np.float64)
    # (token position, slot order, expert, gate) for every routed term
    terms = []
    if cfg.mode == "ec":
        for e in range(cfg.E):
            rows = disp.tok_rows[e, tokens]
            for i, r in enumerate(rows):
                if r >= 0:
                    terms.append((i, e, e, float(disp.row_gate[r])))
    else:
        for i, t in enumerate(tokens):
            for j in range(disp.tok_rows.shape[1]):
                r = disp.tok_rows[t, j]
                if r >= 0:
                    e = int(np.searchsorted(disp.offsets, r, side="right") - 1)
                    terms.append((i, j, e, float(disp.row_gate[r])))
    terms.sort(key=lambda z: (z[0], z[1]))
    # evaluate FFN_e once per expert on the tokens that need it
    contrib: dict[tuple[int, int], np.ndarray] = {}
    by_e: dict[int, list] = {}
    for (i, j, e, g) in terms:
        by_e.setdefault(e, []).append((i, j, g))
    for e, lst in by_e.items():
        rows = x[tokens[[i for (i, _, _) in lst]]]
        out = expert_ffn(rows, w1[e], w2[e], None if w3 is None else w3[e], cfg.act)
        for n, (i, j, g) in enumerate(lst):
            contrib[(i, j)] = g * out[n]
    for (i, j, e, g) in terms:
        y[i] += contrib[(i, j)]
    for s in range(cfg.S):
        ge = cfg.E + s
        y += expert_ffn(x[tokens], w1[ge], w2[ge], None if w3 is None else w3[ge], cfg.act)
    return y


def forward(cfg: OracleConfig, x, w_router, bias, w1, w3, w2, tokens=None,
            state: np.ndarray | None = None) -> OracleResult:
    """The whole layer: routing for every token, outputs for ``tokens``.

    Routing (steps 1-4) always covers all T tokens because capacity,
    keep-fraction and expert choice couple tokens; the FFN and combine
    (step 5) are evaluated only for the requested tokens (all by default).
    """
    logits = router_logits(x, w_router, bias)
    probs, idx, gate, disp = route(cfg, logits, state)
    T = logits.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    y = combine_tokens(cfg, x, w1, w2, w3, disp, tokens)
    return OracleResult(logits, probs, idx, gate, disp, tokens, y)


# --------------------------------------------------------------------------
# backward (training): gradients of L = sum(dy * y) with the routing held fixed
# --------------------------------------------------------------------------
# The pages train these layers (GShard, DeepSeekMoE, DeepSeek-V2/V3 on "MoE技术演进";
# the gating network p = softmax(g) of "Adaptive Mixtures of Local Experts"):
# gradients reach the experts through every kept row, and the router through
# the gate of each kept row (G = p, p / sum of the selected p when
# renormalised, s + b for DeepSeek-V3's bias routing, whose bias is a fixed
# input).  The selection itself (top-k, capacity drops, keep-fraction,
# expert choice, local groups) is piecewise constant in the logits and is held
# fixed, as training frameworks do.  Everything below is float64 with the
# softmax in exact mathematics (the fixed fp32 recipe only serves the integer
# decisions).


@dataclass
class Grads:
    dx: np.ndarray               # [T, d]
    dw_router: np.ndarray        # [E, d]
    dbias: np.ndarray | None     # [E] when a logit bias is given
    dw1: np.ndarray              # [E+S, f, d]
    dw3: np.ndarray | None       # [E+S, f, d] (SwiGLU)
    dw2: np.ndarray              # [E+S, d, f]
    dlogits: np.ndarray | None = None   # [T, E]: dL/d(router logits)


def softmax_f64(logits: np.ndarray) -> np.ndarray:
    """p = exp(l - max l) / sum exp(l - max l) in float64."""
    l = np.asarray(logits, dtype=np.float64)
    e = np.exp(l - l.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def softmax_backward(p: np.ndarray, dp: np.ndarray) -> np.ndarray:
    """dL/dl from dL/dp through p = softmax(l): p * (dp - sum_j p_j dp_j)."""
    return p * (dp - np.sum(p * dp, axis=1, keepdims=True))


def _ffn_parts(xr, w1_e, w2_e, w3_e, act):
    """Forward of one expert on rows xr (float64), keeping what its backward needs."""
    a = xr @ widen(w1_e).T
    if act == "relu":
        h = np.maximum(a, 0.0)
        u = None
    else:
        u = xr @ widen(w3_e).T
        h = a / (1.0 + np.exp(-a)) * u
    return a, u, h, h @ widen(w2_e).T


def _ffn_backward(xr, a, u, h, dyr, w1_e, w2_e, w3_e, act):
    """Backward of FFN_e for rows with output gradients dyr: returns
    (dx rows, dW1, dW3, dW2).  ReLU: dA = dH [A > 0].  SwiGLU: with
    s = sigmoid(A), H = A s U: dA = dH U s (1 + A (1 - s)), dU = dH A s."""
    w2 = widen(w2_e)
    dw2 = dyr.T @ h
    dh = dyr @ w2
    if act == "relu":
        da = dh * (a > 0)
        dw1 = da.T @ xr
        return da @ widen(w1_e), dw1, None, dw2
    s = 1.0 / (1.0 + np.exp(-a))
    da = dh * u * s * (1.0 + a * (1.0 - s))
    du = dh * a * s
    dw1 = da.T @ xr
    dw3 = du.T @ xr
    return da @ widen(w1_e) + du @ widen(w3_e), dw1, dw3, dw2


def _gates_f64(cfg: OracleConfig, logits, disp: Dispatch, idx, state):
    """Gate of every kept row as a float64 function of the logits (the
    selection fixed), and what its backward needs."""
    p = softmax_f64(logits)
    T, E = p.shape
    if cfg.mode == "ec":
        rows_e = np.searchsorted(disp.offsets, np.arange(len(disp.row_token)), side="right") - 1
        return p, p[disp.row_token, rows_e], None
    k = idx.shape[1]
    src = p[np.arange(T)[:, None], idx]                  # gate source of the k selected
    if cfg.rule == "bias":
        src = src + np.asarray(state, np.float64)[idx]
    if cfg.renormalize:
        ssum = src.sum(axis=1, keepdims=True)
        g_sel = src / ssum
    else:
        ssum = None
        g_sel = src
    # gate of each kept row: row of (t, j) is tok_rows[t, j]
    row_gate = np.zeros(len(disp.row_token))
    r = disp.tok_rows
    kept = r >= 0
    row_gate[r[kept]] = g_sel[kept]
    return p, row_gate, (src, ssum, g_sel)


def backward(cfg: OracleConfig, x, w_router, bias, w1, w3, w2, dy, state=None,
             disp: Dispatch | None = None) -> Grads:
    """Gradients of L = sum(dy * y) for the layer's forward, routing fixed.

    ``disp`` is the forward's routing (recomputed here when not given).
    """
    xs = widen(x)
    T, d = xs.shape
    dy = np.asarray(dy, dtype=np.float64)
    logits32 = router_logits(x, w_router, bias)
    probs, idx, gate, disp0 = route(cfg, logits32, state)
    disp = disp0 if disp is None else disp
    logits = widen(x) @ widen(w_router).T + (0.0 if bias is None else widen(bias)[None, :])
    p, row_gate, gparts = _gates_f64(cfg, logits, disp, idx, state)
    E = cfg.E
    G = cfg.E + cfg.S
    f = np.asarray(w1[0]).shape[0]
    dx = np.zeros((T, d))
    dw1 = np.zeros((G, f, d))
    dw3 = np.zeros((G, f, d)) if cfg.act == "swiglu" else None
    dw2 = np.zeros((G, d, f))
    dgate = np.zeros(len(disp.row_token))               # dL / d(gate of each kept row)
    for e in range(G):
        if e < E:
            a0, a1 = int(disp.offsets[e]), int(disp.offsets[e + 1])
            if a1 == a0:
                continue
            toks = disp.row_token[a0:a1].astype(np.int64)
            g = row_gate[a0:a1]
        else:
            toks = np.arange(T)
            g = np.ones(T)
        xr = xs[toks]
        a, u, h, yo = _ffn_parts(xr, w1[e], w2[e], None if w3 is None else w3[e], cfg.act)
        dyr = dy[toks] * g[:, None]
        dxr, gw1, gw3, gw2 = _ffn_backward(xr, a, u, h, dyr, w1[e], w2[e],
                                           None if w3 is None else w3[e], cfg.act)
        np.add.at(dx, toks, dxr)
        dw1[e] += gw1
        dw2[e] += gw2
        if dw3 is not None:
            dw3[e] += gw3
        if e < E:
            dgate[a0:a1] = np.sum(dy[toks] * yo, axis=1)
    # gates -> probabilities
    dp = np.zeros((T, E))
    if cfg.mode == "ec":
        rows_e = np.searchsorted(disp.offsets, np.arange(len(disp.row_token)), side="right") - 1
        np.add.at(dp, (disp.row_token.astype(np.int64), rows_e), dgate)
    else:
        src, ssum, g_sel = gparts
        k = idx.shape[1]
        dg_sel = np.zeros((T, k))
        r = disp.tok_rows
        kept = r >= 0
        dg_sel[kept] = dgate[r[kept]]
        if cfg.renormalize:
            dsrc = (dg_sel - np.sum(dg_sel * g_sel, axis=1, keepdims=True)) / ssum
        else:
            dsrc = dg_sel
        np.add.at(dp, (np.repeat(np.arange(T), k), idx.reshape(-1)), dsrc.reshape(-1))
    # softmax backward, then the router
    dl = softmax_backward(p, dp)
    dx += dl @ widen(w_router)
    return Grads(dx, dl.T @ xs, None if bias is None else dl.sum(axis=0), dw1, dw3, dw2, dl)


def forward_fixed_selection(cfg: OracleConfig, x, w_router, bias, w1, w3, w2, disp: Dispatch,
                            idx, state=None) -> np.ndarray:
    """y [T, d] in float64 for a given selection, gates from the exact
    softmax of the logits (what ``backward`` differentiates)."""
    xs = widen(x)
    T, d = xs.shape
    logits = xs @ widen(w_router).T + (0.0 if bias is None else widen(bias)[None, :])
    _, row_gate, _ = _gates_f64(cfg, logits, disp, idx, state)
    y = np.zeros((T, d))
    for e in range(cfg.E + cfg.S):
        if e < cfg.E:
            a0, a1 = int(disp.offsets[e]), int(disp.offsets[e + 1])
            toks = disp.row_token[a0:a1].astype(np.int64)
            g = row_gate[a0:a1]
        else:
            toks = np.arange(T)
            g = np.ones(T)
        if len(toks) == 0:
            continue
        _, _, _, yo = _ffn_parts(xs[toks], w1[e], w2[e], None if w3 is None else w3[e], cfg.act)
        np.add.at(y, toks, yo * g[:, None])
    return y
