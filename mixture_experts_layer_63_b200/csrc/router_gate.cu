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
// ascending expert order (a shuffle chain, so the order is that of a single
// thread), IEEE division.  Top-k runs k rounds of a warp arg-max on the fp32
// logits: larger value first, lower expert index on ties.
//
// The kernel also counts, per 32-token unit and per rank j, how many tokens
// chose each expert: the histogram of the priority order q = j*T + t that the
// permutation's scan consumes (see permute.cu).
//
// Router logits: for few experts (E <= 32, W_r small enough for shared
// memory) the warp computes them itself from x and W_r in fp32 (fused
// router); otherwise they come from the tcgen05 GEMM in gemm_sm100.cu.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kTokWarps = kUnitTokens;     // one warp per token, one unit per block

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
  int64_t T;
  int d, E, k, n_groups, topk_groups, renormalize, nunit;
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
  // fused router: W_r staged as fp32 in 16-byte groups laid out so that the
  // 32 lanes of a warp read 32 consecutive groups (no bank conflicts):
  // element i of expert e -> group ((e * EPV/4 + (i % EPV) / 4) * nchunk + i / EPV)
  constexpr int EPV = BF16 ? 8 : 4;                      // x elements per 16-byte chunk
  constexpr int GPC = EPV / 4;                           // fp32 groups per chunk
  float4 *s_w = reinterpret_cast<float4 *>(smem + ((hist_ints * 4 + 15) & ~15));
  const int nchunk = P.d / EPV;
  // per-warp buffer of the exponentials, summed in order by lane 0
  float *s_ex = reinterpret_cast<float *>(smem + ((hist_ints * 4 + 15) & ~15) +
                                          (FUSED ? (size_t)E * P.d * 4 : 0)) + warp * E;

  for (int i = threadIdx.x; i < hist_ints; i += blockDim.x) s_hist[i] = 0;
  if (FUSED) {
    const int ngroups = E * P.d / 4;
    for (int gi = threadIdx.x; gi < ngroups; gi += blockDim.x) {
      const int e = gi / (P.d / 4), i0 = (gi - e * (P.d / 4)) * 4;   // 4 consecutive elements
      float4 f;
      if (BF16) {
        const uint2 w = reinterpret_cast<const uint2 *>(P.w_router)[gi];
        f = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
      } else {
        f = reinterpret_cast<const float4 *>(P.w_router)[gi];
      }
      const int c = i0 / EPV, h = (i0 % EPV) / 4;
      s_w[(e * GPC + h) * nchunk + c] = f;
    }
  }
  __syncthreads();

  const int64_t t = (int64_t)blockIdx.x * kTokWarps + warp;
  const bool live = t < P.T;

  // ---- logits of this token: lane l holds experts l + 32 j ----------------
  float l[NV];
  if (FUSED) {
    float acc[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
    if (live) {
      const uint4 *xr = reinterpret_cast<const uint4 *>(P.x) + t * nchunk;
      for (int c = lane; c < nchunk; c += 32) {
        const uint4 xv = xr[c];
        float xf[EPV];
        if (BF16) {
          xf[0] = bf16_lo(xv.x); xf[1] = bf16_hi(xv.x); xf[2 % EPV] = bf16_lo(xv.y); xf[3 % EPV] = bf16_hi(xv.y);
          xf[4 % EPV] = bf16_lo(xv.z); xf[5 % EPV] = bf16_hi(xv.z); xf[6 % EPV] = bf16_lo(xv.w); xf[7 % EPV] = bf16_hi(xv.w);
        } else {
          xf[0] = __uint_as_float(xv.x); xf[1] = __uint_as_float(xv.y);
          xf[2 % EPV] = __uint_as_float(xv.z); xf[3 % EPV] = __uint_as_float(xv.w);
        }
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
          if (e < E) {
            float a = acc[e];
#pragma unroll
            for (int h = 0; h < GPC; ++h) {
              const float4 w = s_w[(e * GPC + h) * nchunk + c];
              a = fmaf(xf[4 * h + 0], w.x, a);
              a = fmaf(xf[4 * h + 1], w.y, a);
              a = fmaf(xf[4 * h + 2], w.z, a);
              a = fmaf(xf[4 * h + 3], w.w, a);
            }
            acc[e] = a;
          }
        }
      }
    }
    float mine = -INFINITY;
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
      if (e < E) {
        float v = acc[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == e) mine = P.bias ? __fadd_rn(v, P.bias[e]) : v;
      }
    }
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
        if (e < E && grp[j] == g) gm = fmaxf(gm, l[j]);
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
        if (ok && (l[j] > bv || (l[j] == bv && e < bi))) {
          bv = l[j];
          bi = e;
        }
      }
      argmax_warp(bv, bi);
      // probability of the chosen expert, from the lane that holds it
      float pv = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j)
        if (j == bi / 32) pv = p[j];
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
      P.hist[((int64_t)r * P.nunit + blockIdx.x) * E + e] = s_hist[i];
    }
  }
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

#ifndef MOE_FUSED_ROUTER_BF16
#define MOE_FUSED_ROUTER_BF16 0
#endif

// fp32 layers: the gate kernel computes the logits (CUDA cores).  bf16 layers
// use the tcgen05 router GEMM.
bool router_is_fused(const moe_config *c) {
  if (c->dtype == MOE_BF16 && !MOE_FUSED_ROUTER_BF16) return false;
  return c->E <= 32 && (size_t)c->E * c->d_model * 4 <= kFusedRouterSmem;
}

cudaError_t launch_route_gate(const moe_config *c, const float *logits_in, float *logits_out,
                              const void *x, const void *w_router, const float *bias, float *probs,
                              int32_t *topk_idx, float *topk_gate, int32_t *hist, cudaStream_t s,
                              int nsplit, int64_t split_stride) {
  GateParams P{};
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
  const int blocks = P.nunit;
  size_t smem = P.hist ? (size_t)P.k * P.E * 4 : 0;
  smem = (smem + 15) & ~(size_t)15;
  smem += (size_t)kTokWarps * c->E * 4;                     // per-warp exponentials
  const int NV = (c->E + 31) / 32;
  if (fused) {
    smem += (size_t)c->E * c->d_model * 4;                  // W_r staged as fp32
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

}  // namespace moe
