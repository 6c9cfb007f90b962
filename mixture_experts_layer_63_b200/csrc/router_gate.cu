// Router and gate: softmax + token-choice top-k (optionally group-limited and
// renormalised), one warp per token.
//
// Softmax gating follows "MoE技术演进", "Adaptive Mixtures of Local Experts"
// (p_i = exp(g_i) / sum_j exp(g_j)); the selector keeps the top-k experts by
// weight; group-limited routing follows DeepSeek-V2 section 3 (choose M
// groups, then top-K inside them).
//
// Lane l of a token's warp holds experts l, l+32, l+64, ...  The arithmetic
// is the fixed fp32 recipe shared with the oracle: m = max, z = l - m (one
// rounded subtraction), exp_det, the denominator summed sequentially in
// ascending expert order (lane 0 adds the exponentials one at a time from
// shared memory, the order of a single thread), IEEE division.  Top-k runs k rounds of a warp arg-max on the fp32
// logits: larger value first, lower expert index on ties.
//
// The kernel also counts, per 32-token unit and per rank j, how many tokens
// chose each expert: the histogram of the priority order q = j*T + t that the
// permutation's scan consumes (see permute.cu).
//
// Router logits: for few experts (E <= 32, W_r small enough for shared
// memory; bf16 up to d_model = 2048) the warp computes them itself from x
// and W_r with fp32 accumulation (fused router: x is read once, no logits
// round trip); otherwise they come from the tcgen05 GEMM in gemm_sm100.cu.
// With the combine folded into the down-projection the kernel also zeroes
// its tokens' rows of y.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kTokWarps = kUnitTokens;     // one warp per token, one unit per block
#ifndef MOE_GATE8
#define MOE_GATE8 1
#endif
#ifndef MOE_GATE_WIDE
#define MOE_GATE_WIDE 1
#endif

struct GateParams {
  const float *logits_in;     // [T, E] (null when the router is fused)
  float *logits_out;          // [T, E] written by the fused router
  const void *x;              // fused router input [T, d]
  const void *w_router;       // fused router weights [E, d]
  const float *bias;          // [E] or null
  float *probs;               // [T, E]
  int32_t *topk_idx;          // [T, k] or null (expert choice)
  float *topk_gate;           // [T, k]
  int32_t *hist;              // [k][nunit][E] or null
  int nsplit;                 // logits_in holds nsplit partial sums ...
  int64_t split_stride;       // ... split_stride floats apart
  const float *state;         // [E] routing bias (rule 1) or utilisation (rule 2)
  int rule;                   // moe_route_rule
  float alpha;                // load-aware coefficient
  int64_t T;
  int d, E, k, n_groups, topk_groups, renormalize, nunit;
  int nbg;                    // 32-token blocks per local group (unit numbering)
  uint4 *y_zero;              // [T, y_vecs] 16-byte vectors set to 0, or null
  int y_vecs;
};

__device__ __forceinline__ void argmax_warp(float &v, int &i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}

__device__ __forceinline__ float max_warp(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One halving step of a warp reduction of N values a lane: the lanes with
// bit `o` set keep the upper N/2 values, the others the lower N/2, each
// adding its partner's copy of the half it keeps.
template <int N, int EMAX>
__device__ __forceinline__ void halve(float (&a)[EMAX], int o, int lane) {
  const bool upper = (lane & o) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = upper ? a[i] : a[N / 2 + i];
    const float keep = upper ? a[N / 2 + i] : a[i];
    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}

// acc + sum over the 8 bf16 pairs of two 16-byte chunks, in element order:
// fma.rn.f32.bf16 multiplies the bf16 operands exactly and rounds once into
// the fp32 accumulator, as fmaf on the widened values does, with no
// widening instructions
__device__ __forceinline__ float dot8_bf16(const uint4 x, const uint4 w, float acc) {
  asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
      "mov.b32 {xl, xh}, %1;\n\tmov.b32 {wl, wh}, %5;\n\t"
      "fma.rn.f32.bf16 %0, xl, wl, %0;\n\tfma.rn.f32.bf16 %0, xh, wh, %0;\n\t"
      "mov.b32 {xl, xh}, %2;\n\tmov.b32 {wl, wh}, %6;\n\t"
      "fma.rn.f32.bf16 %0, xl, wl, %0;\n\tfma.rn.f32.bf16 %0, xh, wh, %0;\n\t"
      "mov.b32 {xl, xh}, %3;\n\tmov.b32 {wl, wh}, %7;\n\t"
      "fma.rn.f32.bf16 %0, xl, wl, %0;\n\tfma.rn.f32.bf16 %0, xh, wh, %0;\n\t"
      "mov.b32 {xl, xh}, %4;\n\tmov.b32 {wl, wh}, %8;\n\t"
      "fma.rn.f32.bf16 %0, xl, wl, %0;\n\tfma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
      : "+f"(acc)
      : "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w));
  return acc;
}

// 16-byte chunk of x or W_r widened to fp32
template <bool BF16>
__device__ __forceinline__ void widen_chunk(const uint4 v, float (&f)[BF16 ? 8 : 4]) {
  if constexpr (BF16) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
  } else {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
}

// NV = slots per lane (ceil(E/32)); FUSED: compute logits from x and W_r
// (requires E <= EMAX <= 32, so NV == 1); BF16: input element type of the
// fused router.
template <int NV, bool FUSED, bool BF16, int EMAX = 32>
__global__ void __launch_bounds__(kTokWarps * 32) route_gate_kernel(const GateParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E = P.E, k = P.k;
  pdl_wait();
  pdl_trigger();
  int *s_hist = reinterpret_cast<int *>(smem);                    // [k][E]
  const int hist_ints = P.hist ? k * E : 0;
  // fused router: W_r as stored, [E][d] in 16-byte chunks
  constexpr int EPV = BF16 ? 8 : 4;                      // elements per 16-byte chunk
  const int nchunk = P.d / EPV;
  uint4 *s_w = reinterpret_cast<uint4 *>(smem + ((hist_ints * 4 + 15) & ~15));
  // per-warp buffer of the exponentials, summed in order by lane 0
  float *s_ex = reinterpret_cast<float *>(s_w + (FUSED ? (size_t)E * nchunk : 0)) + warp * E;

  const int64_t t = (int64_t)blockIdx.x * kTokWarps + warp;
  const bool live = t < P.T;
  if (P.y_zero && live)
    for (int v = lane; v < P.y_vecs; v += 32) P.y_zero[t * P.y_vecs + v] = make_uint4(0u, 0u, 0u, 0u);

  // fused router: this warp's token, lanes split the model dimension (lane l
  // takes chunks l, l + 32, ...); the first NB chunks a lane are in flight
  // while the block stages W_r
  constexpr int NB = EMAX >= 32 ? 2 : 4;
  const uint4 *xr = reinterpret_cast<const uint4 *>(P.x) + (live ? t : 0) * nchunk;
  uint4 xb[NB];
  if (FUSED) {
#pragma unroll
    for (int i = 0; i < NB; ++i) {
      const int c = lane + 32 * i;
      xb[i] = (live && c < nchunk) ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
    }
  }

  for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) s_hist[i] = 0;
  if (FUSED) {
    const uint4 *wg = reinterpret_cast<const uint4 *>(P.w_router);
#pragma unroll 4
    for (int q = threadIdx.x; q < E * nchunk; q += blockDim.x) s_w[q] = wg[q];
  }
  __syncthreads();

  // ---- logits of this token: lane l holds experts l + 32 j ----------------
  float l[NV];
  if (FUSED) {
    // per expert an fp32 sum over this lane's chunks (chunk order, element
    // order inside a chunk), then a halving butterfly over the 32 lanes
    float acc[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < nchunk; c0 += 32 * NB) {
      if (c0 > 0) {
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          const int c = c0 + lane + 32 * i;
          xb[i] = (live && c < nchunk) ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        const int c = c0 + lane + 32 * i;
        if (c >= nchunk) break;
        if constexpr (BF16) {
#pragma unroll
          for (int e = 0; e < EMAX; ++e)
            if (e < E) acc[e] = dot8_bf16(xb[i], s_w[(size_t)e * nchunk + c], acc[e]);
        } else {
          float xf[EPV];
          widen_chunk<BF16>(xb[i], xf);
#pragma unroll
          for (int e = 0; e < EMAX; ++e) {
            if (e < E) {
              float wf[EPV];
              widen_chunk<BF16>(s_w[(size_t)e * nchunk + c], wf);
              float a = acc[e];
#pragma unroll
              for (int h = 0; h < EPV; ++h) a = fmaf(xf[h], wf[h], a);
              acc[e] = a;
            }
          }
        }
      }
    }
    // EMAX values -> one: lane l then holds expert l / (32 / EMAX)
    halve<EMAX, EMAX>(acc, 16, lane);
    if constexpr (EMAX >= 4) halve<EMAX / 2, EMAX>(acc, 8, lane);
    if constexpr (EMAX >= 8) halve<EMAX / 4, EMAX>(acc, 4, lane);
    if constexpr (EMAX >= 16) halve<EMAX / 8, EMAX>(acc, 2, lane);
    if constexpr (EMAX >= 32) halve<EMAX / 16, EMAX>(acc, 1, lane);
    float v = acc[0];
#pragma unroll
    for (int o = 16 / EMAX; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    v = __shfl_sync(0xffffffffu, v, (lane * (32 / EMAX)) & 31);
    float mine = -INFINITY;
    if (lane < E) mine = P.bias ? __fadd_rn(v, P.bias[lane]) : v;
    l[0] = mine;
    if (live && lane < E) P.logits_out[t * E + lane] = mine;
  } else {
    // logits, or partial sums of K parts added in order (then the bias)
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e = lane + 32 * j;
      float v = -INFINITY;
      if (live && e < E) {
        v = P.logits_in[t * E + e];
        for (int sp = 1; sp < P.nsplit; ++sp) v = __fadd_rn(v, P.logits_in[sp * P.split_stride + t * E + e]);
        if (P.bias) v = __fadd_rn(v, P.bias[e]);
        if (P.logits_out) P.logits_out[t * E + e] = v;
      }
      l[j] = v;
    }
  }

  // ---- max, exps, sequential sum, probabilities --------------------------
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < NV; ++j) m = fmaxf(m, l[j]);
  m = max_warp(m);
  float ex[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) ex[j] = (lane + 32 * j < E) ? exp_det(__fsub_rn(l[j], m)) : 0.f;
  // S = sum of the exponentials in ascending expert order, one fp32 add at a time
#pragma unroll
  for (int j = 0; j < NV; ++j)
    if (lane + 32 * j < E) s_ex[lane + 32 * j] = ex[j];
  __syncwarp();
  float S = 0.f;
  if (lane == 0) {
    S = s_ex[0];
#pragma unroll 8
    for (int e = 1; e < E; ++e) S = __fadd_rn(S, s_ex[e]);
  }
  S = __shfl_sync(0xffffffffu, S, 0);
  float p[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    p[j] = __fdiv_rn(ex[j], S);
    if (live && e < E && P.probs) P.probs[t * E + e] = p[j];
  }
  if (P.topk_idx == nullptr) return;          // expert choice: probabilities only

  // ---- selection keys and gate values of the routing rule -----------------
  //   softmax: key = logit, gate = p
  //   bias   : key = p + b_e (one fp32 add), gate = key   (DeepSeek-V3)
  //   load   : key = logit + alpha * (1 - u_e), gate = p   (load-aware top-k)
  float key[NV], gsrc[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    key[j] = l[j];
    gsrc[j] = p[j];
    if (P.rule != 0 && e < E) {
      const float st = P.state[e];
      if (P.rule == 1) {
        key[j] = __fadd_rn(p[j], st);
        gsrc[j] = key[j];
      } else {
        key[j] = __fadd_rn(l[j], __fmul_rn(P.alpha, __fsub_rn(1.0f, st)));
      }
    }
  }

  // ---- group limit: groups of E/n_groups experts, keep the best topk_groups
  uint32_t allowed = 0xffffffffu;
  int grp[NV];                             // group of each slot (0 without a group limit)
  const int gsz = P.n_groups > 0 ? E / P.n_groups : E;
#pragma unroll
  for (int j = 0; j < NV; ++j) grp[j] = (lane + 32 * j) / gsz;
  if (P.n_groups > 0) {
    float my_score = -INFINITY;
    for (int g = 0; g < P.n_groups; ++g) {
      float gm = -INFINITY;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        if (e < E && grp[j] == g) gm = fmaxf(gm, key[j]);
      }
      gm = max_warp(gm);
      if (lane == g) my_score = gm;
    }
    allowed = 0;
    float sv = (lane < P.n_groups) ? my_score : -INFINITY;
    int taken = 0;
    for (int r = 0; r < P.topk_groups; ++r) {
      float v = taken ? -INFINITY : sv;
      int i = (lane < P.n_groups && !taken) ? lane : 0x7fffffff;
      argmax_warp(v, i);
      allowed |= 1u << i;
      if (lane == i) taken = 1;
    }
  }

  // ---- top-k: k rounds of warp arg-max ------------------------------------
  uint32_t taken = 0;          // bit j: slot j of this lane already chosen
  int my_idx = 0;
  float my_gate = 0.f, gsum = 0.f;
  float gates[kMaxTopK];
  int idxs[kMaxTopK];
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    if (r < k) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        const bool ok = e < E && !((taken >> j) & 1u) && ((allowed >> grp[j]) & 1u);
        if (ok && (key[j] > bv || (key[j] == bv && e < bi))) {
          bv = key[j];
          bi = e;
        }
      }
      argmax_warp(bv, bi);
      // gate of the chosen expert, from the lane that holds it
      float pv = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (j == bi / 32) pv = gsrc[j];
      pv = __shfl_sync(0xffffffffu, pv, bi & 31);
      if (lane == (bi & 31)) taken |= 1u << (bi / 32);
      idxs[r] = bi;
      gates[r] = pv;
      gsum = (r == 0) ? pv : __fadd_rn(gsum, pv);
    }
  }
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    if (r < k && lane == r) {
      my_idx = idxs[r];
      my_gate = P.renormalize ? __fdiv_rn(gates[r], gsum) : gates[r];
    }
  }
  if (live && lane < k) {
    P.topk_idx[t * k + lane] = my_idx;
    P.topk_gate[t * k + lane] = my_gate;
    if (P.hist) atomicAdd(&s_hist[lane * E + my_idx], 1);
  }
  if (P.hist) {
    __syncthreads();
    for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) {
      const int r = i / E, e = i - r * E;
      // unit of (rank r, this block): group-major numbering, see unit_grid
      const int g = blockIdx.x / P.nbg, bl = blockIdx.x - g * P.nbg;
      const int64_t u = ((int64_t)g * P.k + r) * P.nbg + bl;
      P.hist[u * E + e] = s_hist[i];
    }
  }
}

// ---------------------------------------------------------------------------
// Gate for more than 32 experts: eight lanes per token, four tokens a warp,
// one 32-token unit a block (256 threads).  Lane s of a token's eight holds
// the contiguous experts [s * EPL, s * EPL + EPL) (EPL >= E / 8), so
//   * the softmax denominator, summed one fp32 add at a time in ascending
//     expert order, runs along the eight lanes in turn (each lane extends
//     the running sum with its own experts and hands it to the next);
//   * maxima and arg-maxima take three shuffle steps;
//   * a token costs a quarter of the instructions of one warp per token.
// Same arithmetic as route_gate_kernel, so the same bits.
// ---------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) gate8_kernel(const GateParams P) {
  __shared__ int s_hist[kMaxTopK * kMaxExperts];          // [k][E] of this unit
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s = lane & 7;                                  // sub-lane of the token
  const int gbase = lane & ~7;
  const int E = P.E, k = P.k;
  pdl_wait();
  pdl_trigger();
  const int64_t t = (int64_t)blockIdx.x * kUnitTokens + warp * 4 + (lane >> 3);
  const bool live = t < P.T;
  const int hist_ints = P.hist ? k * E : 0;
  for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) s_hist[i] = 0;
  if (P.hist) __syncthreads();
  if (P.y_zero && live)
    for (int v = s; v < P.y_vecs; v += 8) P.y_zero[t * P.y_vecs + v] = make_uint4(0u, 0u, 0u, 0u);
  const int e0 = s * EPL;

  // ---- logits: partial sums of the K parts added in order, then the bias --
  float l[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = e0 + j;
    float v = -INFINITY;
    if (live && e < E) {
      v = P.logits_in[t * E + e];
      for (int sp = 1; sp < P.nsplit; ++sp) v = __fadd_rn(v, P.logits_in[sp * P.split_stride + t * E + e]);
      if (P.bias) v = __fadd_rn(v, P.bias[e]);
      if (P.logits_out) P.logits_out[t * E + e] = v;
    }
    l[j] = v;
  }

  // ---- max, exps, the sequential sum, probabilities -------------------------
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPL; ++j) m = fmaxf(m, l[j]);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float p[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) p[j] = (e0 + j < E) ? exp_det(__fsub_rn(l[j], m)) : 0.f;
  float S = 0.f;
#pragma unroll 1
  for (int step = 0; step < 8; ++step) {
    const float prev = __shfl_sync(0xffffffffu, S, gbase | ((step + 7) & 7));
    if (s == step) {
      float acc = prev;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (e0 + j < E) acc = (step == 0 && j == 0) ? p[0] : __fadd_rn(acc, p[j]);
      S = acc;
    }
  }
  S = __shfl_sync(0xffffffffu, S, gbase | 7);
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = e0 + j;
    p[j] = __fdiv_rn(p[j], S);
    if (live && e < E && P.probs) P.probs[t * E + e] = p[j];
  }
  if (P.topk_idx == nullptr) return;          // expert choice: probabilities only

  // ---- selection keys and gate values of the routing rule -------------------
  // in place: l becomes the key, p the gate source
  //   softmax: key = logit, gate = p
  //   bias   : key = p + b_e (one fp32 add), gate = key   (DeepSeek-V3)
  //   load   : key = logit + alpha * (1 - u_e), gate = p   (load-aware top-k)
  if (P.rule != 0) {
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = e0 + j;
      if (e < E) {
        const float st = P.state[e];
        if (P.rule == 1) {
          l[j] = __fadd_rn(p[j], st);
          p[j] = l[j];
        } else {
          l[j] = __fadd_rn(l[j], __fmul_rn(P.alpha, __fsub_rn(1.0f, st)));
        }
      }
    }
  }
  float *key = l, *gsrc = p;

  // ---- group limit: groups of E/n_groups experts, keep the best topk_groups --
  // amask bit j: expert e0 + j may be chosen
  const uint32_t all_mine = EPL >= 32 ? 0xffffffffu : ((1u << EPL) - 1u);
  uint32_t amask = all_mine;
  if (P.n_groups > 0) {
    const int gsz = E / P.n_groups;
    float gs0 = -INFINITY, gs1 = -INFINITY, gs2 = -INFINITY, gs3 = -INFINITY;   // groups s + 8 i
#pragma unroll 1
    for (int g = 0; g < P.n_groups; ++g) {
      const int lo = g * gsz - e0, hi = lo + gsz;          // my slots in group g: [lo, hi)
      float v = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (j >= lo && j < hi && e0 + j < E) v = fmaxf(v, key[j]);
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if ((g & 7) == s) {
        const int i = g >> 3;
        if (i == 0) gs0 = v;
        else if (i == 1) gs1 = v;
        else if (i == 2) gs2 = v;
        else gs3 = v;
      }
    }
    amask = 0;
    uint32_t gtaken = 0;                          // bit i: group s + 8 i chosen
#pragma unroll 1
    for (int r = 0; r < P.topk_groups; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int g = s + 8 * i;
        const float sc = i == 0 ? gs0 : i == 1 ? gs1 : i == 2 ? gs2 : gs3;
        if (g < P.n_groups && !((gtaken >> i) & 1u) && (sc > bv || (sc == bv && g < bi))) {
          bv = sc;
          bi = g;
        }
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if ((bi & 7) == s) gtaken |= 1u << (bi >> 3);
      // my slots of group bi
      const int lo = max(bi * gsz - e0, 0), hi = min(bi * gsz - e0 + gsz, EPL);
      if (lo < hi) {
        const uint32_t upto_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
        amask |= upto_hi & ~((1u << lo) - 1u);
      }
    }
  }

  // ---- top-k: k rounds of an arg-max over the eight lanes --------------------
  // (a loop, not unrolled: the round's result goes to lane r of the eight,
  // so no per-round arrays; keeps the code small for the instruction cache)
  uint32_t taken = 0;                             // bit j: expert e0 + j chosen
  int my_idx = 0;
  float my_gate = 0.f, gsum = 0.f;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY, bg = 0.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = e0 + j;
      const bool ok = e < E && !((taken >> j) & 1u) && ((amask >> j) & 1u);
      if (ok && (key[j] > bv || (key[j] == bv && e < bi))) {
        bv = key[j];
        bi = e;
        bg = gsrc[j];
      }
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const float og = __shfl_xor_sync(0xffffffffu, bg, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
        bg = og;
      }
    }
    if (bi >= e0 && bi < e0 + EPL) taken |= 1u << (bi - e0);
    if (s == r) {
      my_idx = bi;
      my_gate = bg;
    }
    gsum = (r == 0) ? bg : __fadd_rn(gsum, bg);
  }
  if (P.renormalize) my_gate = __fdiv_rn(my_gate, gsum);
  if (live && s < k) {
    P.topk_idx[t * k + s] = my_idx;
    P.topk_gate[t * k + s] = my_gate;
    if (P.hist && my_idx >= 0 && my_idx < E) atomicAdd(&s_hist[s * E + my_idx], 1);
  }
  if (P.hist) {
    __syncthreads();
    for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) {
      const int r = i / E, e = i - r * E;
      // unit of (rank r, this block): group-major numbering, see unit_grid
      const int g = blockIdx.x / P.nbg, bl = blockIdx.x - g * P.nbg;
      const int64_t u = ((int64_t)g * P.k + r) * P.nbg + bl;
      P.hist[u * E + e] = s_hist[i];
    }
  }
}

cudaError_t launch_gate8(const GateParams &P, int blocks, cudaStream_t s) {
  const int epl = (P.E + 7) / 8;
#define MOE_GATE8_CASE(n)                                                          \
  if (epl <= n) return launch_kernel(gate8_kernel<n>, blocks, 256, 0, s, P);
  MOE_GATE8_CASE(8)
  MOE_GATE8_CASE(12)
  MOE_GATE8_CASE(16)
  MOE_GATE8_CASE(20)
  MOE_GATE8_CASE(24)
  MOE_GATE8_CASE(32)
#undef MOE_GATE8_CASE
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Gate for more than 64 experts: a warp a token (lane l holding experts l,
// l + 32, ...), 32 tokens a block, with the two serial parts moved off the
// token's warp:
//   * the softmax denominators: every warp stores its token's exponentials
//     in shared memory, then one warp sums them with a lane per token, each
//     lane adding its token's E values one at a time in ascending expert
//     order (rows padded to E + 1 floats: the 32 lanes read different banks);
//   * the group scores: lane g takes the maximum of group g's keys from the
//     token's row in shared memory, instead of one warp-wide reduction per
//     group.
// Same operations in the same order as route_gate_kernel, so the same bits.
// ---------------------------------------------------------------------------
template <int NV>
__global__ void __launch_bounds__(kTokWarps * 32, 1) gate_wide_kernel(const GateParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int E = P.E, k = P.k, ld = E + 1;
  int *s_hist = reinterpret_cast<int *>(smem);                                // [k][E]
  const int hist_ints = P.hist ? k * E : 0;
  float *s_ex = reinterpret_cast<float *>(smem + ((kMaxTopK * kMaxExperts * 4 + 15) & ~15));
  float *s_key = s_ex + kTokWarps * ld;                                       // [32][E + 1]
  float *s_sum = s_key + kTokWarps * ld;                                      // [32]
  pdl_wait();
  pdl_trigger();
  const int64_t t = (int64_t)blockIdx.x * kTokWarps + warp;
  const bool live = t < P.T;
  for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) s_hist[i] = 0;
  if (P.y_zero && live)
    for (int v = lane; v < P.y_vecs; v += 32) P.y_zero[t * P.y_vecs + v] = make_uint4(0u, 0u, 0u, 0u);

  // ---- logits (K parts added in order, then the bias), max, exponentials ----
  float l[NV], ex[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    float v = -INFINITY;
    if (live && e < E) {
      v = P.logits_in[t * E + e];
      for (int sp = 1; sp < P.nsplit; ++sp) v = __fadd_rn(v, P.logits_in[sp * P.split_stride + t * E + e]);
      if (P.bias) v = __fadd_rn(v, P.bias[e]);
      if (P.logits_out) P.logits_out[t * E + e] = v;
    }
    l[j] = v;
  }
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < NV; ++j) m = fmaxf(m, l[j]);
  m = max_warp(m);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    ex[j] = (live && e < E) ? exp_det(__fsub_rn(l[j], m)) : 0.f;
    if (e < E) s_ex[warp * ld + e] = ex[j];
  }
  __syncthreads();
  // ---- S = sum of a token's exponentials in ascending expert order, one
  //      fp32 add at a time: warp 0, a lane per token ------------------------
  if (warp == 0) {
    const float *row = s_ex + lane * ld;
    float S = row[0];
#pragma unroll 8
    for (int e = 1; e < E; ++e) S = __fadd_rn(S, row[e]);
    s_sum[lane] = S;
  }
  __syncthreads();
  const float S = s_sum[warp];
  float p[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    p[j] = __fdiv_rn(ex[j], S);
    if (live && e < E && P.probs) P.probs[t * E + e] = p[j];
  }
  if (P.topk_idx == nullptr) return;          // expert choice: probabilities only (no barrier follows)

  // ---- selection keys and gate values of the routing rule -------------------
  //   softmax: key = logit, gate = p
  //   bias   : key = p + b_e (one fp32 add), gate = key   (DeepSeek-V3)
  //   load   : key = logit + alpha * (1 - u_e), gate = p   (load-aware top-k)
  float key[NV], gsrc[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    key[j] = l[j];
    gsrc[j] = p[j];
    if (P.rule != 0 && e < E) {
      const float st = P.state[e];
      if (P.rule == 1) {
        key[j] = __fadd_rn(p[j], st);
        gsrc[j] = key[j];
      } else {
        key[j] = __fadd_rn(l[j], __fmul_rn(P.alpha, __fsub_rn(1.0f, st)));
      }
    }
  }

  // ---- group limit: lane g scores group g from the token's keys -------------
  uint32_t allowed = 0xffffffffu;
  const int gsz = P.n_groups > 0 ? E / P.n_groups : E;
  if (P.n_groups > 0) {
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e = lane + 32 * j;
      if (e < E) s_key[warp * ld + e] = key[j];
    }
    __syncwarp();
    float sc = -INFINITY;
    if (lane < P.n_groups) {
      const float *row = s_key + warp * ld + lane * gsz;
      for (int i = 0; i < gsz; ++i) sc = fmaxf(sc, row[i]);
    }
    allowed = 0;
    int gtaken = 0;
    for (int r = 0; r < P.topk_groups; ++r) {
      float v = (lane < P.n_groups && !gtaken) ? sc : -INFINITY;
      int i = (lane < P.n_groups && !gtaken) ? lane : 0x7fffffff;
      argmax_warp(v, i);
      allowed |= 1u << i;
      if (lane == i) gtaken = 1;
    }
  }

  // ---- top-k: k rounds of warp arg-max --------------------------------------
  // open: bit j set while slot j (expert lane + 32 j) exists, is in an
  // allowed group and has not been chosen
  uint32_t open = 0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    if (e < E && ((allowed >> (e / gsz)) & 1u)) open |= 1u << j;
  }
  int my_idx = 0;
  float my_gate = 0.f, gsum = 0.f;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY, bg = 0.f;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e = lane + 32 * j;
      const bool ok = (open >> j) & 1u;
      if (ok && (key[j] > bv || (key[j] == bv && e < bi))) {
        bv = key[j];
        bi = e;
        bg = gsrc[j];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const float og = __shfl_xor_sync(0xffffffffu, bg, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
        bg = og;
      }
    }
    if (lane == (bi & 31)) open &= ~(1u << (bi >> 5));
    if (lane == r) {
      my_idx = bi;
      my_gate = bg;
    }
    gsum = (r == 0) ? bg : __fadd_rn(gsum, bg);
  }
  if (P.renormalize) my_gate = __fdiv_rn(my_gate, gsum);
  if (live && lane < k) {
    P.topk_idx[t * k + lane] = my_idx;
    P.topk_gate[t * k + lane] = my_gate;
    if (P.hist && my_idx >= 0 && my_idx < E) atomicAdd(&s_hist[lane * E + my_idx], 1);
  }
  if (P.hist) {
    __syncthreads();
    for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) {
      const int r = i / E, e = i - r * E;
      // unit of (rank r, this block): group-major numbering, see unit_grid
      const int g = blockIdx.x / P.nbg, bl = blockIdx.x - g * P.nbg;
      const int64_t u = ((int64_t)g * P.k + r) * P.nbg + bl;
      P.hist[u * E + e] = s_hist[i];
    }
  }
}

cudaError_t launch_gate_wide(const GateParams &P, int blocks, cudaStream_t s) {
  const int NV = (P.E + 31) / 32;
  const size_t smem = (size_t)((kMaxTopK * kMaxExperts * 4 + 15) & ~15) +
                      (size_t)2 * kTokWarps * (P.E + 1) * 4 + kTokWarps * 4;
#define MOE_GATE_WIDE_CASE(n)                                                              \
  case n: {                                                                                \
    auto kern = gate_wide_kernel<n>;                                                       \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         (int)smem);                                       \
    if (e != cudaSuccess) return e;                                                        \
    return launch_kernel(kern, blocks, kTokWarps * 32, smem, s, P);                        \
  }
  switch (NV) {
    MOE_GATE_WIDE_CASE(3)
    MOE_GATE_WIDE_CASE(4)
    MOE_GATE_WIDE_CASE(5)
    MOE_GATE_WIDE_CASE(6)
    MOE_GATE_WIDE_CASE(7)
    MOE_GATE_WIDE_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef MOE_GATE_WIDE_CASE
}

cudaError_t launch_nv(int NV, const GateParams &P, int blocks, size_t smem, cudaStream_t s) {
#define MOE_GATE_CASE(n)                                                                       \
  case n: {                                                                                    \
    auto kern = route_gate_kernel<n, false, true>;                                             \
    if (smem > 48 * 1024) {                                                                    \
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                           (int)smem);                                         \
      if (e != cudaSuccess) return e;                                                          \
    }                                                                                          \
    return launch_kernel(kern, blocks, kTokWarps * 32, smem, s, P);                            \
  }
  switch (NV) {
    MOE_GATE_CASE(1)
    MOE_GATE_CASE(2)
    MOE_GATE_CASE(3)
    MOE_GATE_CASE(4)
    MOE_GATE_CASE(5)
    MOE_GATE_CASE(6)
    MOE_GATE_CASE(7)
    MOE_GATE_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef MOE_GATE_CASE
}

}  // namespace

// shared memory of the fused router: W_r as stored
static size_t fused_router_smem(const moe_config *c) {
  return (size_t)c->E * c->d_model * (c->dtype == MOE_BF16 ? 2 : 4);
}

// Few experts (E <= 32) and a W_r that fits shared memory: the gate kernel
// computes the logits itself on CUDA cores, reading x once; otherwise the
// tcgen05 router GEMM (bf16) or a CUDA-core kernel (fp32) runs first.  For
// bf16 the fused form is used up to d = 2048: router + gate 19 vs 24 us on
// the GShard-shaped layer (d = 1024), but 63 vs 50 us on the Mixtral-shaped
// one (d = 4096), where each warp's serial walk along a 8 KB row loses to
// the GEMM.
constexpr int kFusedRouterMaxDBf16 = 2048;

bool router_is_fused(const moe_config *c) {
  if (c->E > 32 || fused_router_smem(c) > kFusedRouterSmem) return false;
  return c->dtype != MOE_BF16 || c->d_model <= kFusedRouterMaxDBf16;
}

cudaError_t launch_route_gate(const moe_config *c, const float *logits_in, float *logits_out,
                              const void *x, const void *w_router, const float *bias,
                              const float *state, float *probs, int32_t *topk_idx, float *topk_gate,
                              int32_t *hist, cudaStream_t s, int nsplit, int64_t split_stride,
                              void *y_zero) {
  GateParams P{};
  P.y_zero = static_cast<uint4 *>(y_zero);
  P.y_vecs = (int)((int64_t)c->d_model * (c->dtype == MOE_BF16 ? 2 : 4) / 16);
  P.rule = c->mode == MOE_TOKEN_CHOICE ? c->route_rule : MOE_ROUTE_SOFTMAX;
  P.state = state;
  P.alpha = c->route_alpha;
  P.nsplit = nsplit < 1 ? 1 : nsplit;
  P.split_stride = split_stride;
  const bool tc = c->mode == MOE_TOKEN_CHOICE;
  const bool fused = logits_in == nullptr;
  P.logits_in = logits_in;
  P.logits_out = logits_out;
  P.x = x;
  P.w_router = w_router;
  P.bias = bias;
  P.probs = probs;
  P.topk_idx = tc ? topk_idx : nullptr;
  P.topk_gate = tc ? topk_gate : nullptr;
  P.hist = tc ? hist : nullptr;
  P.T = c->T;
  P.d = c->d_model;
  P.E = c->E;
  P.k = tc ? c->k : 0;
  P.n_groups = c->n_groups;
  P.topk_groups = c->topk_groups;
  P.renormalize = c->renormalize;
  P.nunit = (int)((c->T + kUnitTokens - 1) / kUnitTokens);
  P.nbg = unit_grid(c).nbg;
  const int blocks = P.nunit;
  size_t smem = P.hist ? (size_t)P.k * P.E * 4 : 0;
  smem = (smem + 15) & ~(size_t)15;
  smem += (size_t)kTokWarps * c->E * 4;                     // per-warp exponentials
  const int NV = (c->E + 31) / 32;
  if (fused) {
    smem += fused_router_smem(c);                           // W_r as stored
    const bool bf = c->dtype == MOE_BF16;
    auto kern = c->E <= 8    ? (bf ? route_gate_kernel<1, true, true, 8> : route_gate_kernel<1, true, false, 8>)
                : c->E <= 16 ? (bf ? route_gate_kernel<1, true, true, 16> : route_gate_kernel<1, true, false, 16>)
                             : (bf ? route_gate_kernel<1, true, true, 32> : route_gate_kernel<1, true, false, 32>);
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    return launch_kernel(kern, blocks, kTokWarps * 32, smem, s, P);
  }
  // 33 to 64 experts: eight lanes a token (8 experts a lane, 60 registers);
  // beyond that a warp a token, whose registers stay few enough for 32
  // warps an SM (measured: DeepSeekMoE's 64 experts route 50 vs 65 us; 160
  // experts 95 vs 83 us and 256 experts 191 vs 108 us the other way).
  // MOE_GATE8=0 at build time: a warp a token throughout.
  if (NV > 1 && MOE_GATE8 && c->E <= 64) return launch_gate8(P, blocks, s);
  // more than 64 experts: a warp a token, sums and group scores off the warp
  if (NV > 2 && MOE_GATE_WIDE) return launch_gate_wide(P, blocks, s);
  return launch_nv(NV, P, blocks, smem, s);
}

}  // namespace moe

namespace moe {
namespace {
// fp32 router on CUDA cores: one warp per token, lanes split the model
// dimension (fp32 layers with more than 32 experts or a large W_r).
__global__ void __launch_bounds__(256) router_f32_kernel(const float *__restrict__ x,
                                                         const float *__restrict__ w,
                                                         const float *__restrict__ bias,
                                                         float *__restrict__ logits, int64_t T,
                                                         int d, int E) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  const float *xr = x + t * d;
  for (int e = 0; e < E; ++e) {
    const float *wr = w + (int64_t)e * d;
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) acc = fmaf(xr[i], wr[i], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logits[t * E + e] = bias ? __fadd_rn(acc, bias[e]) : acc;
  }
}
}  // namespace

cudaError_t launch_router_f32(const moe_config *c, const float *x, const float *w,
                              const float *bias, float *logits, cudaStream_t s) {
  const int warps = 8;
  const int64_t blocks = (c->T + warps - 1) / warps;
  return launch_kernel(router_f32_kernel, (unsigned)blocks, warps * 32, 0, s, x, w, bias, logits,
                       c->T, c->d_model, c->E);
}

namespace {
// DeepSeek-V3 bias update: b_e -= gamma when c_e * E > T * k, += gamma when
// c_e * E < T * k (exact integer load test), unchanged at the mean.
__global__ void bias_update_kernel(const int32_t *__restrict__ counts, float *__restrict__ bias,
                                   int E, int64_t Tk, float gamma) {
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int64_t load = (int64_t)counts[e] * E;
    if (load > Tk) bias[e] = __fsub_rn(bias[e], gamma);
    else if (load < Tk) bias[e] = __fadd_rn(bias[e], gamma);
  }
}
}  // namespace

cudaError_t launch_bias_update(const moe_config *c, const int32_t *counts, float *bias, float gamma,
                               cudaStream_t s) {
  return launch_kernel(bias_update_kernel, 1, 256, 0, s, counts, bias, c->E, c->T * (int64_t)c->k,
                       gamma);
}

}  // namespace moe
