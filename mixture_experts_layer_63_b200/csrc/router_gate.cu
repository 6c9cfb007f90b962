// Router logits (fp32 CUDA-core path) and the gate: softmax + token-choice
// top-k, optionally group-limited and renormalised.
//
// Softmax gating follows "MoE技术演进", "Adaptive Mixtures of Local Experts"
// (p_i = exp(g_i) / sum_j exp(g_j)); the selector keeps the top-k experts by
// weight; group-limited routing follows DeepSeek-V2 section 3 (choose M
// groups, then top-K inside them).  The bf16 router logits come from the
// tcgen05 GEMM in gemm_sm100.cu; this file's gate kernel serves both dtypes.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

// ---------------------------------------------------------------------------
// fp32 router: one warp per token, lanes split the model dimension.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_f32_kernel(const float *__restrict__ x,
                                                         const float *__restrict__ w,
                                                         const float *__restrict__ bias,
                                                         float *__restrict__ logits, int64_t T,
                                                         int d, int E) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float *xr = x + t * d;
  for (int e = 0; e < E; ++e) {
    const float *wr = w + (int64_t)e * d;
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) acc = fmaf(xr[i], wr[i], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) logits[t * E + e] = bias ? acc + bias[e] : acc;
  }
}

cudaError_t launch_router_f32(const moe_config *c, const float *x, const float *w,
                              const float *bias, float *logits, cudaStream_t s) {
  const int warps = 8;
  const int64_t blocks = (c->T + warps - 1) / warps;
  router_f32_kernel<<<(unsigned)blocks, warps * 32, 0, s>>>(x, w, bias, logits, c->T, c->d_model,
                                                            c->E);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Gate: one thread per token.
//   1. m = max_e l; with group limits, group maxima and the chosen groups
//      (larger maximum first, lower group on ties);
//   2. top-k over the allowed experts on the fp32 logits: strictly larger
//      first, lower expert index on ties (candidates visited in ascending
//      index, and an equal value never displaces an earlier one);
//   3. S = sum_e exp_det(l_e - m), sequential in ascending e, fp32;
//   4. p_e = exp_det(l_e - m) / S (IEEE division); gates = p of the chosen
//      experts, or p / (their sum in rank order) when renormalising.
// ---------------------------------------------------------------------------
// Insert (v, i) into a list sorted by value, descending.  Candidates arrive
// in ascending index order, so an equal value stays behind the ones already
// listed; once inserted, every later entry shifts down one place.
__device__ __forceinline__ void topk_insert(float v, int i, float (&tv)[kMaxTopK],
                                            int (&ti)[kMaxTopK]) {
  bool shifting = false;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    const bool better = shifting || (ti[j] < 0) || (v > tv[j]);
    shifting = better;
    const float ov = tv[j];
    const int oi = ti[j];
    tv[j] = better ? v : ov;
    ti[j] = better ? i : oi;
    v = better ? ov : v;
    i = better ? oi : i;
  }
}

__global__ void __launch_bounds__(128) gate_kernel(const float *__restrict__ logits,
                                                   float *__restrict__ probs,
                                                   int32_t *__restrict__ topk_idx,
                                                   float *__restrict__ topk_gate, int64_t T, int E,
                                                   int k, int n_groups, int topk_groups,
                                                   int renormalize) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const float *l = logits + t * E;

  float m = -INFINITY;
  for (int e = 0; e < E; ++e) m = fmaxf(m, l[e]);

  // allowed-group mask (all groups when the limit is off)
  uint32_t allowed = 0xffffffffu;
  int gsz = E;
  if (n_groups > 0) {
    gsz = E / n_groups;
    float gv[kMaxTopK];
    int gi[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) { gv[j] = -INFINITY; gi[j] = -1; }
    for (int g = 0; g < n_groups; ++g) {
      float gm = -INFINITY;
      for (int e = g * gsz; e < (g + 1) * gsz; ++e) gm = fmaxf(gm, l[e]);
      topk_insert(gm, g, gv, gi);
    }
    allowed = 0;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < topk_groups && gi[j] >= 0) allowed |= 1u << gi[j];
  }

  if (topk_idx != nullptr) {
    float tv[kMaxTopK];
    int ti[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) { tv[j] = -INFINITY; ti[j] = -1; }
    for (int e = 0; e < E; ++e) {
      if (n_groups > 0 && !((allowed >> (e / gsz)) & 1u)) continue;
      const float v = l[e];
      if (ti[kMaxTopK - 1] >= 0 && !(v > tv[kMaxTopK - 1])) continue;   // cannot enter the top list
      topk_insert(v, e, tv, ti);
    }
    // probabilities of the chosen experts, same arithmetic as below
    float S = 0.f;
    for (int e = 0; e < E; ++e) S = (e == 0) ? exp_det(__fsub_rn(l[0], m)) : __fadd_rn(S, exp_det(__fsub_rn(l[e], m)));
    float g[kMaxTopK];
    float gs = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        g[j] = __fdiv_rn(exp_det(__fsub_rn(l[ti[j]], m)), S);
        gs = (j == 0) ? g[j] : __fadd_rn(gs, g[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        topk_idx[t * k + j] = ti[j];
        topk_gate[t * k + j] = renormalize ? __fdiv_rn(g[j], gs) : g[j];
      }
    }
    if (probs != nullptr) {
      float *p = probs + t * E;
      for (int e = 0; e < E; ++e) p[e] = __fdiv_rn(exp_det(__fsub_rn(l[e], m)), S);
    }
  } else {
    float S = 0.f;
    for (int e = 0; e < E; ++e) S = (e == 0) ? exp_det(__fsub_rn(l[0], m)) : __fadd_rn(S, exp_det(__fsub_rn(l[e], m)));
    float *p = probs + t * E;
    for (int e = 0; e < E; ++e) p[e] = __fdiv_rn(exp_det(__fsub_rn(l[e], m)), S);
  }
}

cudaError_t launch_gate(const moe_config *c, const float *logits, float *probs, int32_t *topk_idx,
                        float *topk_gate, cudaStream_t s) {
  const int threads = 128;
  const int64_t blocks = (c->T + threads - 1) / threads;
  const bool tc = c->mode == MOE_TOKEN_CHOICE;
  gate_kernel<<<(unsigned)blocks, threads, 0, s>>>(logits, probs, tc ? topk_idx : nullptr,
                                                   tc ? topk_gate : nullptr, c->T, c->E, c->k,
                                                   c->n_groups, c->topk_groups, c->renormalize);
  return cudaGetLastError();
}

}  // namespace moe
