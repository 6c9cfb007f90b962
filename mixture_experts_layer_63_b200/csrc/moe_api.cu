// C ABI of libmoe.so (declared in include/moe.h): argument validation,
// workspace layout and the launch sequence of each entry point.  All
// arithmetic of the layer runs in the kernels of the other files.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <unordered_map>

#include <nvtx3/nvToolsExt.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

// NVTX range around an entry point or a phase of moe_forward (host-side
// markers for profilers; header-only, inert when no tool is attached).
struct Range {
  explicit Range(const char *name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range &) = delete;
  Range &operator=(const Range &) = delete;
};

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Expert capacity (GShard section 1 of "MoE技术演进": C = O(N/E) tokens per
// expert; per local group of N/G tokens with group dispatching):
// C = ceil(cf * k * Tg / E) for the fp32 factor cf, Tg = T / G tokens per
// group, evaluated exactly: cf = m * 2^s with m a 24-bit integer, so
// C = ceil(m * k * Tg * 2^s / E) in 128-bit integers.  Clamped to Tg (an
// expert takes at most one assignment per token); 0 = unlimited.
int64_t capacity_rows(const moe_config *c) {
  if (c->mode != MOE_TOKEN_CHOICE || !(c->capacity_factor > 0.0f)) return 0;
  const int64_t Tg = c->local_groups > 1 ? c->T / c->local_groups : c->T;
  int ex = 0;
  const double mant = frexp((double)c->capacity_factor, &ex);      // cf = mant * 2^ex
  const uint64_t m = (uint64_t)ldexp(mant, 24);                     // exact: fp32 has 24 bits
  const int s = ex - 24;                                            // cf = m * 2^s
  unsigned __int128 num = (unsigned __int128)m * (uint64_t)c->k * (uint64_t)Tg;
  unsigned __int128 den = (uint64_t)c->E;
  if (s >= 0) {
    if (s > 60) return Tg;                      // cf >= 2^60: far above Tg
    num <<= s;
  } else {
    if (-s > 100) return num > 0 ? 1 : 0;       // 0 < value < 1: the ceiling is 1
    den <<= -s;
  }
  const unsigned __int128 q = (num + den - 1) / den;
  return q >= (unsigned __int128)Tg ? Tg : (int64_t)q;
}

moe_status validate(const moe_config *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->d_model < 1 || c->d_ff < 1 || c->E < 1 || c->S < 0) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->act != MOE_ACT_RELU && c->act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (c->mode != MOE_TOKEN_CHOICE && c->mode != MOE_EXPERT_CHOICE) return MOE_ERR_INVALID_ARG;
  if (c->renormalize != 0 && c->renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (c->keep_den < 0 || c->keep_num < 0 || (c->keep_den > 0 && c->keep_num > c->keep_den) ||
      (c->keep_den == 0 && c->keep_num != 0))
    return MOE_ERR_INVALID_ARG;
  if (c->n_groups < 0 || c->topk_groups < 0) return MOE_ERR_INVALID_ARG;
  if (c->route_rule < MOE_ROUTE_SOFTMAX || c->route_rule > MOE_ROUTE_LOAD || c->reserved != 0)
    return MOE_ERR_INVALID_ARG;
  if (!(c->route_alpha == c->route_alpha)) return MOE_ERR_INVALID_ARG;       // NaN
  if (!std::isfinite(c->capacity_factor)) return MOE_ERR_INVALID_ARG;
  const bool capped = c->capacity_factor > 0.0f;
  if (c->local_groups < 0) return MOE_ERR_INVALID_ARG;
  if (c->local_groups > 1) {
    // GShard local groups: capacity dispatch of contiguous 32-token-aligned groups
    if (c->mode != MOE_TOKEN_CHOICE || !capped) return MOE_ERR_INVALID_ARG;
    if (c->T % c->local_groups != 0) return MOE_ERR_INVALID_ARG;
    if ((c->T / c->local_groups) % kUnitTokens != 0) return MOE_ERR_UNSUPPORTED;
  }
  if (c->mode == MOE_TOKEN_CHOICE) {
    if (c->k < 1 || c->k > c->E) return MOE_ERR_INVALID_ARG;
    if (capped && c->keep_den > 0) return MOE_ERR_INVALID_ARG;            // exclusive drop rules
    if (c->n_groups > 0) {
      if (c->E % c->n_groups != 0 || c->topk_groups < 1 || c->topk_groups > c->n_groups)
        return MOE_ERR_INVALID_ARG;
      if ((int64_t)c->topk_groups * (c->E / c->n_groups) < c->k) return MOE_ERR_INVALID_ARG;
    } else if (c->topk_groups != 0) {
      return MOE_ERR_INVALID_ARG;
    }
    if (c->T * (int64_t)c->k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->ec_capacity < 1 || c->ec_capacity > c->T) return MOE_ERR_INVALID_ARG;
    if (c->n_groups != 0 || c->topk_groups != 0 || capped || c->keep_den > 0 ||
        c->renormalize || c->route_rule != MOE_ROUTE_SOFTMAX)
      return MOE_ERR_INVALID_ARG;
    if ((int64_t)c->E * c->ec_capacity > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  }
  // limits of this build
  if (c->E > kMaxExperts || c->S > 8) return MOE_ERR_UNSUPPORTED;
  if (c->mode == MOE_TOKEN_CHOICE && (c->k > kMaxTopK || c->n_groups > 32 || c->topk_groups > 8))
    return MOE_ERR_UNSUPPORTED;
  if (c->T > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_BF16) {
    if (c->d_model % 64 != 0 || c->d_ff % 64 != 0) return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d_model % 4 != 0) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

// MOE_FUSED_GATHER=1 at build time: moe_forward's up-projection gathers the
// routed rows of x itself (16-byte cp.async copies in the tile kernels;
// measured slower than the gather kernel, so off by default).
#ifndef MOE_FUSED_GATHER
#define MOE_FUSED_GATHER 0
#endif
static bool forward_gathers(const moe_config *c, int64_t rows_cap) {
  (void)rows_cap;
  return c->dtype == MOE_BF16 && MOE_FUSED_GATHER;
}

#ifndef MOE_DOWN_REVERSE
#define MOE_DOWN_REVERSE 0
#endif

WsLayout make_layout(const moe_config *c) {
  WsLayout L{};
  const int64_t T = c->T;
  const int E = c->E, S = c->S;
  const bool tc = c->mode == MOE_TOKEN_CHOICE;
  const int k = tc ? c->k : 0;
  const size_t es = elem_size(c);
  L.rows_cap = tc ? T * k : (int64_t)E * c->ec_capacity;
  L.rows_total = L.rows_cap + (int64_t)S * T;
  L.tok_rows_len = tc ? T * k : (int64_t)E * T;
  L.nunit = (int)((T + kUnitTokens - 1) / kUnitTokens);
  const int64_t hist_ints = tc ? (int64_t)k * L.nunit * E : 0;
  const bool keepfrac = tc && capacity_rows(c) == 0 && c->keep_den > 0;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.err = take(kCtrlBytes);
  L.hist = take((size_t)hist_ints * 4);
  L.base = take((size_t)(tc ? unit_grid(c).nb * E : 0) * 4);           // per-block unit totals
  L.cnt_off = take((size_t)(E + 1) * 4);
  L.kept = take((size_t)E * 4);
  L.sorted_q = take(keepfrac ? (size_t)T * k * 4 : 0);
  L.probs_t = take(tc ? 0 : (size_t)E * T * 4);
  L.permute_end = o;
  const int ks = (c->dtype == MOE_BF16 && !router_is_fused(c) && !router_tc_used(c)) ? router_ksplit(c) : 1;
  L.logits_part = take(ks > 1 ? (size_t)ks * T * E * 4 : 0);
  L.sk_part = take(c->dtype == MOE_BF16 ? (size_t)kSkSlots * kSkSlotFloats * 4 : 0);
  L.step_end = o;
  L.logits = take((size_t)T * E * 4);
  L.probs = take((size_t)T * E * 4);
  L.topk_idx = take((size_t)T * k * 4);
  L.topk_gate = take((size_t)T * k * 4);
  L.counts = take((size_t)E * 4);
  L.offsets = take((size_t)(E + 1) * 4);
  L.n_dropped = take(4);
  L.tok_rows = take((size_t)L.tok_rows_len * 4);
  L.row_token = take((size_t)L.rows_cap * 4);
  L.row_gate = take((size_t)L.rows_cap * 4);
  // moe_forward's x_perm: bf16 layers gather inside the up-projection GEMM
  const bool fused_gather = forward_gathers(c, L.rows_cap);
  L.x_perm = take(fused_gather ? 0 : (size_t)L.rows_cap * c->d_model * es);
  L.h = take((size_t)L.rows_total * c->d_ff * es);
  L.y_rows = take((size_t)L.rows_total * c->d_model * es);     // rows in the layer dtype
  L.total = o;
  L.x_stage = take((size_t)T * c->d_model * es);
  L.y_stage = take((size_t)T * c->d_model * es);
  L.host_total = o;
  return L;
}

static moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

static moe_status check_ws(const WsLayout &L, const void *ws, size_t ws_bytes, size_t need) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  (void)L;
  return MOE_OK;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The combine folded into the down-projection (moe_forward): with at most
// two rows a token (k + S <= 2, token choice), the gate zeroes y and the
// down-projection's epilogue adds each gated bf16 row into its token's row
// of y with bf16 vector reductions.  Two bf16 additions onto 0 commute, so
// the result is the same in whatever order the rows arrive: y = bf16(r1 +
// r2), as the combine kernel computes it.  No y_rows, no combine launch.
#ifndef MOE_FOLD_COMBINE
#define MOE_FOLD_COMBINE 1
#endif
static bool combine_folded(const moe_config *c) {
  return MOE_FOLD_COMBINE && c->mode == MOE_TOKEN_CHOICE && c->dtype == MOE_BF16 && c->k + c->S <= 2;
}

// ---- step bodies, shared by the step entry points and moe_forward ----------
// y_zero non-null: the gate also sets y to 0 (the folded combine)
static cudaError_t run_route(const moe_config *c, const WsLayout &L, char *ws, const void *x,
                             const void *w_router, const float *bias, const float *state,
                             float *logits, float *probs, int32_t *topk_idx, float *topk_gate,
                             cudaStream_t s, void *y_zero = nullptr) {
  int32_t *hist = c->mode == MOE_TOKEN_CHOICE ? reinterpret_cast<int32_t *>(ws + L.hist) : nullptr;
  if (router_is_fused(c))
    return launch_route_gate(c, nullptr, logits, x, w_router, bias, state, probs, topk_idx,
                             topk_gate, hist, s, 1, 0, y_zero);
  // bf16: the tcgen05 router GEMM with the gate in its epilogue (logits
  // written only when the caller wants them)
  if (router_tc_used(c))
    return launch_router_tc(c, x, w_router, bias, state, logits, probs, topk_idx, topk_gate, hist,
                            y_zero, reinterpret_cast<uint32_t *>(ws + L.err), s);
  cudaError_t e;
  if (c->dtype == MOE_F32) {
    e = launch_router_f32(c, static_cast<const float *>(x), static_cast<const float *>(w_router),
                          bias, logits, s);
  } else {
    GroupedGemm g{};
    g.epi = kEpiStoreF32;
    g.K = c->d_model;
    g.N = c->E;
    g.a = x;
    g.a_rows = c->T;
    g.a_static = x;
    g.a_static_rows = c->T;
    g.b = w_router;
    g.b3 = nullptr;
    g.b_rows = c->E;
    g.offsets = nullptr;
    g.n_routed = 0;
    g.n_static = 1;
    g.rows_static = c->T;
    g.a_static_base = 0;
    g.a_static_stride = 0;
    g.out_static_base = 0;
    g.max_routed_rows = 0;
    g.err = reinterpret_cast<uint32_t *>(ws + L.err);
    const int ks = router_ksplit(c);
    if (ks > 1) {
      // K split over more CTAs; the gate adds the parts in order, then the bias
      float *parts = reinterpret_cast<float *>(ws + L.logits_part);
      g.out = parts;
      g.ksplit = ks;
      g.split_stride = c->T * c->E;
      e = launch_grouped_gemm(g, s);
      if (e != cudaSuccess) return e;
      return launch_route_gate(c, parts, logits, nullptr, nullptr, bias, state, probs, topk_idx,
                               topk_gate, hist, s, ks, c->T * c->E, y_zero);
    }
    g.out = logits;
    g.bias = bias;
    e = launch_grouped_gemm(g, s);
  }
  if (e != cudaSuccess) return e;
  return launch_route_gate(c, logits, nullptr, nullptr, nullptr, nullptr, state, probs, topk_idx,
                           topk_gate, hist, s, 1, 0, y_zero);
}

// row_token non-null (bf16): the up-projection gathers the routed rows of x
// itself and x_perm is not read.  y_add non-null (bf16): the folded combine,
// the down-projection adds row r into y_add[add_rows[r]] (zeroed by the gate)
// instead of writing y_rows.
static cudaError_t run_ffn(const moe_config *c, const WsLayout &L, char *ws, const void *x,
                           const void *x_perm, const int32_t *offsets, const float *row_gate,
                           const void *w1, const void *w3, const void *w2, void *h, void *y_rows,
                           cudaStream_t s, const int32_t *row_token = nullptr,
                           void *y_add = nullptr, const int32_t *add_rows = nullptr) {
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + L.err);
  if (c->dtype == MOE_F32)
    return launch_ffn_f32(c, L, err, static_cast<const float *>(x),
                          static_cast<const float *>(x_perm), offsets, row_gate,
                          static_cast<const float *>(w1), static_cast<const float *>(w3),
                          static_cast<const float *>(w2), static_cast<float *>(h),
                          static_cast<float *>(y_rows), s);
  const bool swiglu = c->act == MOE_ACT_SWIGLU;
  GroupedGemm up{};
  up.epi = swiglu ? kEpiSwiglu : kEpiRelu;
  up.K = c->d_model;
  up.N = c->d_ff;
  up.a = row_token ? x : x_perm;
  up.a_rows = row_token ? c->T : L.rows_cap;
  up.gather_rows = row_token;
  up.gather_src = row_token ? x : nullptr;
  up.src_rows = c->T;
  up.a_static = x;
  up.a_static_rows = c->T;
  up.b = w1;
  up.b3 = swiglu ? w3 : nullptr;
  up.b_rows = (int64_t)(c->E + c->S) * c->d_ff;
  up.offsets = offsets;
  up.n_routed = c->E;
  up.n_static = c->S;
  up.rows_static = c->T;
  up.a_static_base = 0;
  up.a_static_stride = 0;
  up.out_static_base = L.rows_cap;
  up.max_routed_rows = L.rows_cap;
  up.out = h;
  up.out_rows = L.rows_total;
  up.sk_part = reinterpret_cast<float *>(ws + L.sk_part);
  up.sk_flags = reinterpret_cast<int *>(ws + L.err + kSkFlagsOffset);
  up.err = err;
  cudaError_t e = launch_grouped_gemm(up, s);
  if (e != cudaSuccess) return e;
  GroupedGemm dn{};
  dn.epi = y_add ? kEpiScaleAdd : kEpiScale;
  dn.K = c->d_ff;
  dn.N = c->d_model;
  dn.a = h;
  dn.a_rows = L.rows_total;
  dn.a_static = h;
  dn.a_static_rows = L.rows_total;
  dn.b = w2;
  dn.b3 = nullptr;
  dn.b_rows = (int64_t)(c->E + c->S) * c->d_model;
  dn.offsets = offsets;
  dn.n_routed = c->E;
  dn.n_static = c->S;
  dn.rows_static = c->T;
  dn.a_static_base = L.rows_cap;
  dn.a_static_stride = c->T;
  dn.out_static_base = L.rows_cap;
  dn.max_routed_rows = L.rows_cap;
  dn.out = y_add ? y_add : y_rows;
  dn.out_rows = y_add ? 0 : L.rows_total;
  dn.add_rows = y_add ? add_rows : nullptr;
  dn.src_rows = c->T;
  dn.row_gate = row_gate;
  // the last groups' activations are the ones still in L2 when the
  // up-projection ends: start the down-projection there
  dn.reverse = MOE_DOWN_REVERSE;
  dn.sk_part = up.sk_part;
  dn.sk_flags = up.sk_flags;
  dn.err = err;
  return launch_grouped_gemm(dn, s);
}

// ---- backward ----------------------------------------------------------------
static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

struct BwLayout {
  size_t x_perm;            // the routed rows of x, when the forward left no x_perm
  size_t dy_perm, au, dau, dx_rows, kseg, kseg_r, dyT, hT, dauT, xT, dgate, dg_part, dl, dl_pad,
      dlT, xTr, wrT, dx_router, total;
  int64_t kp_max, Ep, Tp;
  int fw;
  int dg_nt;                // 256-column N-tiles of the dact GEMM (pieces of a gate gradient)
};

static BwLayout make_bw_layout(const moe_config *c, const WsLayout &L) {
  BwLayout B{};
  const int64_t T = c->T, d = c->d_model, f = c->d_ff;
  const int G = c->E + c->S;
  B.fw = (int)(c->act == MOE_ACT_SWIGLU ? 2 * f : f);
  B.kp_max = round_up(L.rows_total + 64 * (int64_t)G, 64);
  B.Ep = round_up(c->E, 64);
  B.Tp = round_up(T, 64);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  B.x_perm = take(forward_gathers(c, L.rows_cap) ? (size_t)L.rows_cap * d * 2 : 0);
  B.dy_perm = take((size_t)L.rows_cap * d * 2);
  B.au = take((size_t)L.rows_total * B.fw * 2);
  B.dau = take((size_t)L.rows_total * B.fw * 2);
  B.dx_rows = take((size_t)L.rows_total * d * 4);
  B.kseg = take((size_t)(G + 1) * 4);
  B.kseg_r = take(2 * 4);
  B.dyT = take((size_t)d * B.kp_max * 2);
  B.hT = take((size_t)f * B.kp_max * 2);
  B.dauT = take((size_t)B.fw * B.kp_max * 2);
  B.xT = take((size_t)d * B.kp_max * 2);
  B.dgate = take((size_t)L.rows_cap * 4);
  B.dg_nt = (int)((f + 255) / 256);
  B.dg_part = take((size_t)L.rows_cap * B.dg_nt * 4);
  B.dl = take((size_t)T * c->E * 4);
  B.dl_pad = take((size_t)T * B.Ep * 2);
  B.dlT = take((size_t)c->E * B.Tp * 2);
  B.xTr = take((size_t)d * B.Tp * 2);
  B.wrT = take((size_t)d * B.Ep * 2);
  B.dx_router = take((size_t)T * d * 4);
  B.total = o;
  return B;
}

static cudaError_t run_backward(const moe_config *c, const WsLayout &L, const BwLayout &B,
                                const char *ws_c, char *bw, const void *x, const void *w_router,
                                const float *state, const void *w1, const void *w3, const void *w2,
                                const void *dy, float *dx, float *dw_router, float *dbias,
                                float *dw1, float *dw3, float *dw2, cudaStream_t s) {
  char *ws = const_cast<char *>(ws_c);          // GEMM scratch and error word of the forward's workspace
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + L.err);
  float *sk_part = reinterpret_cast<float *>(ws + L.sk_part);
  int *sk_flags = reinterpret_cast<int *>(ws + L.err + kSkFlagsOffset);
  const int64_t T = c->T, d = c->d_model, f = c->d_ff;
  const int E = c->E, S = c->S, G = E + S;
  const bool swiglu = c->act == MOE_ACT_SWIGLU;
  const float *probs = reinterpret_cast<const float *>(ws + L.probs);
  const int32_t *topk_idx = reinterpret_cast<const int32_t *>(ws + L.topk_idx);
  const int32_t *offsets = reinterpret_cast<const int32_t *>(ws + L.offsets);
  const int32_t *tok_rows = reinterpret_cast<const int32_t *>(ws + L.tok_rows);
  const int32_t *row_token = reinterpret_cast<const int32_t *>(ws + L.row_token);
  const float *row_gate = reinterpret_cast<const float *>(ws + L.row_gate);
  const void *h = ws + L.h;
  const bool fused_gather = forward_gathers(c, L.rows_cap);
  void *dy_perm = bw + B.dy_perm;
  void *au = bw + B.au, *dau = bw + B.dau;
  float *dx_rows = reinterpret_cast<float *>(bw + B.dx_rows);
  int32_t *kseg = reinterpret_cast<int32_t *>(bw + B.kseg);
  int32_t *kseg_r = reinterpret_cast<int32_t *>(bw + B.kseg_r);
  float *dgate = reinterpret_cast<float *>(bw + B.dgate);
  float *dl = reinterpret_cast<float *>(bw + B.dl);
  float *dx_router = reinterpret_cast<float *>(bw + B.dx_router);
  cudaError_t e;
#define MOE_TRY(x_)            \
  do {                         \
    e = (x_);                  \
    if (e != cudaSuccess) return e; \
  } while (0)

  // 1. the routed rows of x: the forward's x_perm, or gathered here when the
  // forward's up-projection read them from x itself
  const void *xp = ws + L.x_perm;
  if (fused_gather) {
    MOE_TRY(launch_gather_bf16_rows(x, bw + B.x_perm, row_token, offsets, E, T, (int)d, L.rows_cap,
                                    err, s));
    xp = bw + B.x_perm;
  }
  // 2. pre-activations recomputed: A (| U) [rows_total][fw]
  GroupedGemm up{};
  up.epi = swiglu ? kEpiPreSwiglu : kEpiPreRelu;
  up.K = (int)d;
  up.N = (int)f;
  up.a = xp;
  up.a_rows = L.rows_cap;
  up.src_rows = T;
  up.a_static = x;
  up.a_static_rows = T;
  up.b = w1;
  up.b3 = swiglu ? w3 : nullptr;
  up.b_rows = (int64_t)G * f;
  up.offsets = offsets;
  up.n_routed = E;
  up.n_static = S;
  up.rows_static = T;
  up.out_static_base = L.rows_cap;
  up.max_routed_rows = L.rows_cap;
  up.out = au;
  up.sk_part = sk_part;
  up.sk_flags = sk_flags;
  up.err = err;
  MOE_TRY(launch_grouped_gemm(up, s));

  // 3. dY of the routed rows (ungated; the gate is applied in the epilogue)
  MOE_TRY(launch_gather_bf16_rows(dy, dy_perm, row_token, offsets, E, T, (int)d, L.rows_cap, err, s));

  // 4. dA (| dU) = act'(A, U) * (g * dY . W2)
  GroupedGemm dh{};
  dh.epi = swiglu ? kEpiDActSwiglu : kEpiDActRelu;
  dh.K = (int)d;
  dh.N = (int)f;
  dh.a = dy_perm;
  dh.a_rows = L.rows_cap;
  dh.a_static = dy;
  dh.a_static_rows = T;
  dh.b = w2;                       // W2 [G][d][f] read as [K = d][N = f]
  dh.b_mn = 1;
  dh.b_krows = d;
  dh.b_rows = (int64_t)G * d;
  dh.offsets = offsets;
  dh.n_routed = E;
  dh.n_static = S;
  dh.rows_static = T;
  dh.out_static_base = L.rows_cap;
  dh.max_routed_rows = L.rows_cap;
  dh.out = dau;
  dh.aux = au;
  dh.aux_ld = B.fw;
  dh.dg_part = reinterpret_cast<float *>(bw + B.dg_part);
  dh.dg_nt = B.dg_nt;
  dh.aux2 = h;                     // the forward's activations (SwiGLU's gate-gradient pieces)
  dh.aux2_ld = f;
  dh.row_gate = row_gate;
  dh.sk_part = sk_part;
  dh.sk_flags = sk_flags;
  dh.err = err;
  MOE_TRY(launch_grouped_gemm(dh, s));

  // 5. dX rows = [dA | dU] . [W1 ; W3]   (fp32 rows)
  GroupedGemm dxg{};
  dxg.epi = kEpiStoreF32;
  dxg.K = B.fw;
  dxg.N = (int)d;
  dxg.a = dau;
  dxg.a_rows = L.rows_total;
  dxg.a_static = dau;
  dxg.a_static_rows = L.rows_total;
  dxg.a_static_base = L.rows_cap;
  dxg.a_static_stride = T;
  dxg.b = w1;                      // W1 (| W3) [G][f][d] read as [K = f (+ f)][N = d]
  dxg.b3 = swiglu ? w3 : nullptr;
  dxg.b_mn = 1;
  dxg.b_krows = f;
  dxg.b_kb_split = (int)(f / 64);
  dxg.b_rows = (int64_t)G * f;
  dxg.offsets = offsets;
  dxg.n_routed = E;
  dxg.n_static = S;
  dxg.rows_static = T;
  dxg.out_static_base = L.rows_cap;
  dxg.max_routed_rows = L.rows_cap;
  dxg.out = dx_rows;
  dxg.sk_part = sk_part;
  dxg.sk_flags = sk_flags;
  dxg.err = err;
  MOE_TRY(launch_grouped_gemm(dxg, s));

  // 6-8. gate gradients, router logits gradient dl, bias gradient
  MOE_TRY(launch_gate_grad(reinterpret_cast<const float *>(bw + B.dg_part), B.dg_nt, offsets, E,
                           L.rows_cap, dgate, s));
  MOE_TRY(launch_router_grad(c, probs, topk_idx, tok_rows, dgate, state, dl, s));
  if (dbias) MOE_TRY(launch_bias_grad(dl, T, E, dbias, s));

  // 9. router term of dx: dl [T, E] . W_r [E, d] (K padded to 64 with zeros)
  MOE_TRY(launch_pad_f32_bf16(dl, bw + B.dl_pad, T, E, (int)B.Ep, s));
  MOE_TRY(cudaMemsetAsync(bw + B.wrT, 0, (size_t)d * B.Ep * 2, s));
  MOE_TRY(launch_transpose_bf16(w_router, bw + B.wrT, E, (int)d, d, B.Ep, 1, 0, 0, 0, s));
  GroupedGemm rx{};
  rx.epi = kEpiStoreF32;
  rx.K = (int)B.Ep;
  rx.N = (int)d;
  rx.a = bw + B.dl_pad;
  rx.a_rows = T;
  rx.a_static = bw + B.dl_pad;
  rx.a_static_rows = T;
  rx.b = bw + B.wrT;
  rx.b_rows = d;
  rx.n_routed = 0;
  rx.n_static = 1;
  rx.rows_static = T;
  rx.out = dx_router;
  rx.ksplit = 1;
  rx.err = err;
  MOE_TRY(launch_grouped_gemm(rx, s));

  // 10. dx = its dX rows + shared rows + the router term
  MOE_TRY(launch_dx_finish(c, L.rows_cap, dx_rows, tok_rows, dx_router, dx, s));

  // 11. router weights: dW_r = dl^T . x  (one K group over the tokens)
  MOE_TRY(launch_transpose_f32_bf16(dl, bw + B.dlT, (int)T, E, (int)B.Tp, B.Tp, s));
  MOE_TRY(cudaMemsetAsync(bw + B.xTr, 0, (size_t)d * B.Tp * 2, s));
  MOE_TRY(launch_transpose_bf16(x, bw + B.xTr, (int)T, (int)d, d, B.Tp, 1, 0, 0, 0, s));
  MOE_TRY(launch_seg_offsets(nullptr, 0, 1, T, kseg_r, s));
  GroupedGemm rw{};
  rw.epi = kEpiStoreF32;
  rw.kgroup = 1;
  rw.M = E;
  rw.K = (int)B.Tp;
  rw.N = (int)d;
  rw.a = bw + B.dlT;
  rw.a_rows = B.Tp;
  rw.b = bw + B.xTr;
  rw.b_rows = d;
  rw.n_routed = 0;
  rw.n_static = 1;
  rw.kseg = kseg_r;
  rw.out = dw_router;
  rw.err = err;
  MOE_TRY(launch_grouped_gemm(rw, s));

  // 12. expert weights: each expert contracts over its own rows (K groups)
  MOE_TRY(launch_seg_offsets(offsets, E, S, T, kseg, s));
  MOE_TRY(launch_transpose_segments(dy, d, row_token, row_gate, 0, 0, T, T, offsets, kseg, E, G,
                                    (int)d, B.kp_max, bw + B.dyT, err, s));
  MOE_TRY(launch_transpose_segments(h, f, nullptr, nullptr, L.rows_cap, T, T, L.rows_total, offsets,
                                    kseg, E, G, (int)f, B.kp_max, bw + B.hT, err, s));
  MOE_TRY(launch_transpose_segments(dau, B.fw, nullptr, nullptr, L.rows_cap, T, T, L.rows_total,
                                    offsets, kseg, E, G, B.fw, B.kp_max, bw + B.dauT, err, s));
  MOE_TRY(launch_transpose_segments(x, d, row_token, nullptr, 0, 0, T, T, offsets, kseg, E, G,
                                    (int)d, B.kp_max, bw + B.xT, err, s));
  GroupedGemm w2g{};
  w2g.epi = kEpiStoreF32;
  w2g.kgroup = 1;
  w2g.M = (int)d;
  w2g.K = (int)B.kp_max;
  w2g.N = (int)f;
  w2g.a = bw + B.dyT;
  w2g.a_rows = B.kp_max;
  w2g.b = bw + B.hT;
  w2g.b_rows = f;
  w2g.n_routed = 0;
  w2g.n_static = G;
  w2g.kseg = kseg;
  w2g.out = dw2;
  w2g.err = err;
  MOE_TRY(launch_grouped_gemm(w2g, s));
  GroupedGemm w1g = w2g;
  w1g.M = B.fw;
  w1g.N = (int)d;
  w1g.a = bw + B.dauT;
  w1g.b = bw + B.xT;
  w1g.b_rows = d;
  w1g.out = dw1;
  w1g.out2 = swiglu ? dw3 : nullptr;
  w1g.split_m = (int)f;
  MOE_TRY(launch_grouped_gemm(w1g, s));
#undef MOE_TRY
  return cudaSuccess;
}

}  // namespace moe

using namespace moe;

// Per-workspace ordering of moe_forward_host calls: the input copy of a call
// waits for the previous forward on the workspace (which read the staged x),
// the forward for the previous output copy (which read the staged y).
namespace {
struct HostEvents {
  cudaEvent_t in_done = nullptr, fwd_done = nullptr, out_done = nullptr;
};
std::mutex g_host_mutex;
std::unordered_map<const void *, HostEvents> g_host_events;

cudaError_t host_events(const void *ws, HostEvents *out) {
  std::lock_guard<std::mutex> lock(g_host_mutex);
  HostEvents &h = g_host_events[ws];
  for (cudaEvent_t *e : {&h.in_done, &h.fwd_done, &h.out_done}) {
    if (*e == nullptr) {
      const cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
      if (r != cudaSuccess) {
        *e = nullptr;
        return r;
      }
    }
  }
  *out = h;
  return cudaSuccess;
}
}  // namespace

extern "C" {

moe_status moe_query_sizes(const moe_config *cfg, moe_sizes *out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  const moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  out->rows_cap = L.rows_cap;
  out->rows_total = L.rows_total;
  out->tok_rows_len = L.tok_rows_len;
  out->step_workspace = L.step_end;
  out->workspace = L.total;
  out->capacity = capacity_rows(cfg);
  out->permute_workspace = L.permute_end;
  out->host_workspace = L.host_total;
  return MOE_OK;
}

// the routing state array is required exactly when the rule reads it
static bool state_ok(const moe_config *c, const float *state) {
  return c->route_rule == MOE_ROUTE_SOFTMAX || state != nullptr;
}

moe_status moe_route(const moe_config *cfg, const void *x, const void *w_router, const float *bias,
                     const float *route_state, float *logits, float *probs, int32_t *topk_idx,
                     float *topk_gate, void *ws, size_t ws_bytes, moe_stream_t stream) {
  Range range("moe_route");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.step_end)) != MOE_OK) return st;
  const bool tc = cfg->mode == MOE_TOKEN_CHOICE;
  if (!x || !w_router || !logits || !probs || (tc && (!topk_idx || !topk_gate)))
    return MOE_ERR_INVALID_ARG;
  if (!state_ok(cfg, route_state)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(logits) || !aligned16(probs))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(run_route(cfg, L, static_cast<char *>(ws), x, w_router, bias, route_state,
                               logits, probs, topk_idx, topk_gate,
                               reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_gate(const moe_config *cfg, const float *logits, const float *route_state,
                    float *probs, int32_t *topk_idx, float *topk_gate, void *ws, size_t ws_bytes,
                    moe_stream_t stream) {
  Range range("moe_gate");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.step_end)) != MOE_OK) return st;
  const bool tc = cfg->mode == MOE_TOKEN_CHOICE;
  if (!logits || !probs || (tc && (!topk_idx || !topk_gate))) return MOE_ERR_INVALID_ARG;
  if (!state_ok(cfg, route_state)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_route_gate(cfg, logits, nullptr, nullptr, nullptr, nullptr, route_state,
                                       probs, topk_idx, topk_gate, nullptr,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_route_bias_update(const moe_config *cfg, const int32_t *counts, float *route_bias,
                                 float gamma, moe_stream_t stream) {
  const moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->mode != MOE_TOKEN_CHOICE || !counts || !route_bias) return MOE_ERR_INVALID_ARG;
  if (!(gamma == gamma)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_bias_update(cfg, counts, route_bias, gamma,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                       const float *topk_gate, const float *probs, int32_t *counts, int32_t *offsets,
                       int32_t *tok_rows, int32_t *row_token, float *row_gate, void *x_perm,
                       int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream) {
  Range range("moe_permute");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.step_end)) != MOE_OK) return st;
  const bool tc = cfg->mode == MOE_TOKEN_CHOICE;
  const bool keepfrac = tc && capacity_rows(cfg) == 0 && cfg->keep_den > 0;
  if (!x || !counts || !offsets || !tok_rows || !row_token || !row_gate || !x_perm || !n_dropped)
    return MOE_ERR_INVALID_ARG;
  if (tc && (!topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if ((!tc || keepfrac) && !probs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_permute(cfg, L, static_cast<char *>(ws), false, x, topk_idx, topk_gate, probs,
                                    counts, offsets, tok_rows, row_token, row_gate, x_perm,
                                    n_dropped, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const moe_config *cfg, const void *x, const void *x_perm,
                          const int32_t *offsets, const float *row_gate, const void *w1,
                          const void *w3, const void *w2, void *h, void *y_rows, void *ws,
                          size_t ws_bytes, moe_stream_t stream) {
  Range range("moe_expert_ffn");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.step_end)) != MOE_OK) return st;
  const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
  if (!x || !x_perm || !offsets || !row_gate || !w1 || !w2 || !h || !y_rows || (swiglu && !w3))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm) || !aligned16(w1) || !aligned16(w2) || !aligned16(h) ||
      !aligned16(y_rows) || (swiglu && !aligned16(w3)))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(run_ffn(cfg, L, static_cast<char *>(ws), x, x_perm, offsets, row_gate, w1, w3,
                             w2, h, y_rows, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_config *cfg, const void *y_rows, const int32_t *tok_rows, void *y,
                       moe_stream_t stream) {
  Range range("moe_combine");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  if (!y_rows || !tok_rows || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_rows) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = make_layout(cfg);
  return cuda_status(launch_combine(cfg, L.rows_cap, y_rows, tok_rows, y,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

static moe_status forward_impl(const moe_config *cfg, const void *x, const void *w_router,
                               const float *bias, const float *state, const void *w1,
                               const void *w3, const void *w2, void *y, int32_t *counts_out,
                               void *ws, size_t ws_bytes, void *const *events,
                               moe_stream_t stream) {
  Range range("moe_forward");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
  if (!x || !w_router || !w1 || !w2 || !y || (swiglu && !w3)) return MOE_ERR_INVALID_ARG;
  if (!state_ok(cfg, state)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w1) || !aligned16(w2) || !aligned16(y) ||
      (swiglu && !aligned16(w3)))
    return MOE_ERR_INVALID_ARG;
  const bool fold = combine_folded(cfg);
  {
    // y is written from the first kernel on (folded combine): it may not overlap x
    const uintptr_t xb = reinterpret_cast<uintptr_t>(x), yb = reinterpret_cast<uintptr_t>(y);
    const uintptr_t n = (uintptr_t)cfg->T * (uintptr_t)cfg->d_model * elem_size(cfg);
    if (xb < yb + n && yb < xb + n) return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *w = static_cast<char *>(ws);
  float *logits = reinterpret_cast<float *>(w + L.logits);
  float *probs = reinterpret_cast<float *>(w + L.probs);
  int32_t *topk_idx = reinterpret_cast<int32_t *>(w + L.topk_idx);
  float *topk_gate = reinterpret_cast<float *>(w + L.topk_gate);
  int32_t *counts = reinterpret_cast<int32_t *>(w + L.counts);
  int32_t *offsets = reinterpret_cast<int32_t *>(w + L.offsets);
  int32_t *n_dropped = reinterpret_cast<int32_t *>(w + L.n_dropped);
  int32_t *tok_rows = reinterpret_cast<int32_t *>(w + L.tok_rows);
  int32_t *row_token = reinterpret_cast<int32_t *>(w + L.row_token);
  float *row_gate = reinterpret_cast<float *>(w + L.row_gate);
  void *x_perm = w + L.x_perm;
  void *h = w + L.h;
  void *y_rows = w + L.y_rows;
  auto mark = [&](int i) -> cudaError_t {
    if (events && events[i]) return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
    return cudaSuccess;
  };
  cudaError_t e = mark(0);
  if (e == cudaSuccess) {
    Range r("route");
    // (the forward's logits have no reader: the fused router skips them)
    e = run_route(cfg, L, w, x, w_router, bias, state, router_tc_used(cfg) ? nullptr : logits, probs,
                  topk_idx, topk_gate, s, fold ? y : nullptr);
  }
  if (e == cudaSuccess) e = mark(1);
  // token choice: the gate wrote the unit histogram into the workspace.
  // bf16: the up-projection gathers the rows of x itself (no x_perm)
  const bool fused_gather = forward_gathers(cfg, L.rows_cap);
  if (e == cudaSuccess) {
    Range r("permute");
    e = launch_permute(cfg, L, w, cfg->mode == MOE_TOKEN_CHOICE, x, topk_idx, topk_gate, probs,
                       counts, offsets, tok_rows, row_token, row_gate, x_perm, n_dropped, s,
                       !fused_gather);
  }
  if (e == cudaSuccess) e = mark(2);
  if (e == cudaSuccess) {
    Range r("expert_ffn");
    e = run_ffn(cfg, L, w, x, x_perm, offsets, row_gate, w1, w3, w2, h, y_rows, s,
                fused_gather ? row_token : nullptr, fold ? y : nullptr, row_token);
  }
  if (e == cudaSuccess) e = mark(3);
  if (e == cudaSuccess && !fold) {
    Range r("combine");
    e = launch_combine(cfg, L.rows_cap, y_rows, tok_rows, y, s);
  }
  if (e == cudaSuccess) e = mark(4);
  if (e == cudaSuccess && counts_out)
    e = cudaMemcpyAsync(counts_out, counts, (size_t)cfg->E * 4, cudaMemcpyDeviceToDevice, s);
  return cuda_status(e);
}

moe_status moe_forward(const moe_config *cfg, const void *x, const void *w_router,
                       const float *bias, const float *route_state, const void *w1, const void *w3,
                       const void *w2, void *y, int32_t *counts_out, void *ws, size_t ws_bytes,
                       moe_stream_t stream) {
  return forward_impl(cfg, x, w_router, bias, route_state, w1, w3, w2, y, counts_out, ws, ws_bytes,
                      nullptr, stream);
}


moe_status moe_forward_host(const moe_config *cfg, const void *x_host, const void *w_router,
                            const float *bias, const float *route_state, const void *w1,
                            const void *w3, const void *w2, void *y_host, int32_t *counts_out,
                            void *ws, size_t ws_bytes, moe_stream_t stream, moe_stream_t copy_in,
                            moe_stream_t copy_out) {
  Range range("moe_forward_host");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.host_total)) != MOE_OK) return st;
  if (!x_host || !y_host) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t cin = copy_in ? reinterpret_cast<cudaStream_t>(copy_in) : s;
  cudaStream_t cout = copy_out ? reinterpret_cast<cudaStream_t>(copy_out) : s;
  HostEvents ev;
  if (host_events(ws, &ev) != cudaSuccess) return MOE_ERR_CUDA;
  char *w = static_cast<char *>(ws);
  const size_t bytes = (size_t)cfg->T * cfg->d_model * elem_size(cfg);
  cudaError_t e = cudaStreamWaitEvent(cin, ev.fwd_done, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(w + L.x_stage, x_host, bytes, cudaMemcpyHostToDevice, cin);
  if (e == cudaSuccess) e = cudaEventRecord(ev.in_done, cin);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev.in_done, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev.out_done, 0);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  st = forward_impl(cfg, w + L.x_stage, w_router, bias, route_state, w1, w3, w2, w + L.y_stage,
                    counts_out, ws, ws_bytes, nullptr, stream);
  if (st != MOE_OK) return st;
  e = cudaEventRecord(ev.fwd_done, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, ev.fwd_done, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(y_host, w + L.y_stage, bytes, cudaMemcpyDeviceToHost, cout);
  if (e == cudaSuccess) e = cudaEventRecord(ev.out_done, cout);
  return cuda_status(e);
}

moe_status moe_forward_timed(const moe_config *cfg, const void *x, const void *w_router,
                             const float *bias, const float *route_state, const void *w1,
                             const void *w3, const void *w2, void *y, int32_t *counts_out,
                             void *ws, size_t ws_bytes, void *const *events, moe_stream_t stream) {
  return forward_impl(cfg, x, w_router, bias, route_state, w1, w3, w2, y, counts_out, ws, ws_bytes,
                      events, stream);
}

moe_status moe_query_backward_size(const moe_config *cfg, size_t *bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  const WsLayout L = make_layout(cfg);
  *bytes = make_bw_layout(cfg, L).total;
  return MOE_OK;
}

moe_status moe_backward(const moe_config *cfg, const void *x, const void *w_router,
                        const float *bias, const float *route_state, const void *w1,
                        const void *w3, const void *w2, const void *dy, float *dx, float *dw_router,
                        float *dbias, float *dw1, float *dw3, float *dw2, const void *ws,
                        size_t ws_bytes, void *bws, size_t bws_bytes, moe_stream_t stream) {
  Range range("moe_backward");
  moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  const WsLayout L = make_layout(cfg);
  if ((st = check_ws(L, ws, ws_bytes, L.total)) != MOE_OK) return st;
  const BwLayout B = make_bw_layout(cfg, L);
  if ((st = check_ws(L, bws, bws_bytes, B.total)) != MOE_OK) return st;
  const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
  if (!x || !w_router || !w1 || !w2 || !dy || !dx || !dw_router || !dw1 || !dw2 ||
      (swiglu && (!w3 || !dw3)) || (bias && !dbias))
    return MOE_ERR_INVALID_ARG;
  if (!state_ok(cfg, route_state)) return MOE_ERR_INVALID_ARG;
  for (const void *p : {x, w_router, w1, w2, dy, static_cast<const void *>(dx),
                        static_cast<const void *>(dw_router), static_cast<const void *>(dw1),
                        static_cast<const void *>(dw2)})
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (swiglu && (!aligned16(w3) || !aligned16(dw3))) return MOE_ERR_INVALID_ARG;
  return cuda_status(run_backward(cfg, L, B, static_cast<const char *>(ws), static_cast<char *>(bws),
                                  x, w_router, route_state, w1, w3, w2, dy, dx, dw_router, dbias,
                                  dw1, dw3, dw2, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_check_device_errors(void *ws, size_t ws_bytes, moe_stream_t stream, uint32_t *flags) {
  if (!ws || ws_bytes < 4) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&word, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  // after a device error the stream-K flags may be left set: clear the block
  if (word != 0 && cudaMemset(ws, 0, std::min(ws_bytes, kCtrlBytes)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (flags) *flags = word;
  if (word & kErrTimeout) return MOE_ERR_TIMEOUT;
  if (word & kErrBadIndex) return MOE_ERR_DEVICE_CHECK;
  return MOE_OK;
}

moe_status moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ws || ws_bytes < 256) return MOE_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, std::min(ws_bytes, kCtrlBytes),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_workspace_set_wait_limit(void *ws, size_t ws_bytes, uint64_t limit_ns,
                                        moe_stream_t stream) {
  if (!ws || ws_bytes < kCtrlBytes || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return MOE_ERR_INVALID_ARG;
  // from host memory: the value is staged before the call returns
  return cuda_status(cudaMemcpyAsync(static_cast<char *>(ws) + kWaitLimitOffset, &limit_ns,
                                     sizeof(limit_ns), cudaMemcpyHostToDevice,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "device-side index check failed";
    case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

uint64_t moe_kernel_launches(void) { return moe::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
