// Router GEMM with the gate in its epilogue (bf16 layers, up to 256 experts).
//
// The router is a linear map followed by a softmax ("大语言模型并行策略（七）：
// 专家并行", section "Mixture of Experts (MoE)"; p_i = exp(g_i) / sum_j exp(g_j)
// of "Adaptive Mixtures of Local Experts" in "MoE技术演进"), then the top-k
// selector, optionally limited to the best groups of experts (DeepSeek-V2
// section 3 of "MoE技术演进").  Here the whole chain is one kernel: the
// logits l = x W_r^T (+ b) never leave the chip.
//
// A cluster of KS CTAs (KS = 2 or 4) owns 256 tokens; CTA c of the cluster
// contracts K part c (k-blocks [c K/(64 KS), (c+1) K/(64 KS))) for all 256:
//   warp 0      TMA producer: per 64-wide k-block, x rows [r0, r0+128) and
//               [r0+128, r0+256) (two 16 KB boxes) and all Np rows of W_r
//               (Np = E rounded up to 16; rows >= E arrive as zeros), 128-byte
//               swizzle, into a ring of stages
//   warp 1      MMA issuer: two tcgen05.mma (M = 128, N = Np, K = 16) per
//               K step, one per 128-token half, sharing the W_r tile, fp32
//               accumulators in TMEM columns [0, Np) and [256, 256 + Np)
//   warp 2      TMEM allocation (512 columns)
// Each CTA reads its x rows once and W_r once per 256 tokens (half the W_r
// traffic of 128-token tiles).  Then, all warps:
//   1. cluster barrier: every CTA is done with its stage ring;
//   2. each CTA sends, for every other CTA j, its partial sums of the
//      256 / KS tokens that j owns (tcgen05.ld, then st.shared::cluster
//      into j's receive slots, which reuse j's stage ring; blocks of 32
//      rows x 4 columns, so that every warp-wide store covers 512
//      contiguous bytes);
//   3. cluster barrier; the owner adds the KS parts in K order (its own part
//      straight from TMEM), then the bias: its tokens' fp32 logits, in
//      shared memory;
//   4. the gate, eight lanes a token (16 warps, 64 tokens a pass), lane s
//      holding the contiguous experts [s EPL, s EPL + EPL): max,
//      exp_det(l - max), the denominator summed one fp32 add at a time in
//      ascending expert order along the eight lanes, IEEE division, the
//      routing rule's keys, group scores (max key of a group) and the best
//      topk_groups groups, k rounds of arg-max (lower expert index on
//      ties), renormalisation, the per-unit histogram of the permutation
//      and, with the combine folded, zeroed rows of y.
// The gate's arithmetic is the same sequence of fp32 operations as the
// separate gate kernels (router_gate.cu) and the oracle, so from the same
// logits the routing is bit-identical.
//
// Every wait is bounded.  A CTA whose wait ran out sets the timeout bit,
// drains its own copies and MMAs and still takes both cluster barriers (no
// CTA of the cluster is left waiting); its outputs are then not valid.
#include <math.h>

#include <algorithm>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100_ptx.cuh"

#ifndef MOE_ROUTER_TC
#define MOE_ROUTER_TC 1
#endif

namespace moe {
namespace {

constexpr int kRtThreads = 512;
constexpr int kRtTile = 256;              // tokens per cluster
constexpr int kRtBK = 64;                 // K per k-block (one 128-byte swizzled row)
constexpr int kRtMaxStages = 6;
constexpr int kRtLanes = 8;               // gate lanes a token
constexpr uint32_t kRtHalfBytes = 128 * kRtBK * 2;     // one 128-token x box: 16 KB
constexpr size_t kRtSmemCap = 227 * 1024 - 2048;        // dynamic shared memory we may ask for
// Partial sums and logits in shared memory: blocks of [32 rows][4 columns]
// (one row group, one 4-column group), padded to 132 floats so that the
// eight lanes of a token, reading eight different blocks, hit different
// banks.  A warp's 16-byte accesses to one block are 512 contiguous bytes.
constexpr int kRtBlk = 132;

struct RtParams {
  const float *bias;          // [E] or null
  float *logits_out;          // [T, E] or null
  float *probs;               // [T, E] or null
  int32_t *topk_idx;          // [T, k]; null: expert choice (probabilities only)
  float *topk_gate;           // [T, k]
  int32_t *hist;              // [units][E] or null
  const float *state;         // [E] routing bias (rule 1) or utilisation (rule 2)
  int rule;
  float alpha;
  int64_t T;
  int K, E, Np, k, n_groups, topk_groups, renormalize, nbg, nunit;
  int ks;                     // CTAs a cluster (K parts)
  int stages;
  uint4 *y_zero;              // [T, y_vecs] set to 0, or null
  int y_vecs;
  uint32_t *err;
};

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}

// Offset (floats) of element (row r, column e) in a [rows][NC * 32] matrix
// stored as kRtBlk-float blocks ordered (row group, 32-column chunk,
// 4-column group): the layout of the receive slots and of the logits.
__device__ __forceinline__ int blk_off(int r, int e, int NC) {
  return (((r >> 5) * NC + (e >> 5)) * 8 + ((e >> 2) & 7)) * kRtBlk + (r & 31) * 4 + (e & 3);
}

// ---------------------------------------------------------------------------
// The gate of one token, eight lanes a token (lanes 8i .. 8i+7 of the warp),
// lane s holding experts [s EPL, s EPL + EPL).  `lg` is the block matrix of
// logits in shared memory, `r` the token's row in it (the group limit
// overwrites the token's logits with its selection keys).  All 32 lanes of
// the warp call it together (shuffles over the full warp).
// ---------------------------------------------------------------------------
template <int EPL>
__device__ __forceinline__ void gate8(const RtParams &P, float *lg, int r, int NC, int64_t t,
                                      bool live, int s, int lane, int *hist_blk) {
  static_assert(EPL % 4 == 0 && EPL <= 32, "four-aligned slots, one 32-bit mask");
  const int E = P.E, k = P.k;
  const int e0 = s * EPL;
  const int gb = lane & ~7;
  const int mine = max(0, min(EPL, E - e0));          // my experts
  float l[EPL];
#pragma unroll
  for (int j = 0; j < EPL; j += 4) {
    const float4 v = *reinterpret_cast<const float4 *>(lg + blk_off(r, e0 + j, NC));
    l[j] = j < mine ? v.x : -INFINITY;
    l[j + 1] = j + 1 < mine ? v.y : -INFINITY;
    l[j + 2] = j + 2 < mine ? v.z : -INFINITY;
    l[j + 3] = j + 3 < mine ? v.w : -INFINITY;
  }
  // ---- softmax: max, exps, the sequential sum, probabilities ----------------
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < EPL; ++j) m = fmaxf(m, l[j]);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // slots past E hold -inf: exp_det gives exactly 0 there, and adding 0 to
  // the running sum leaves it unchanged, so neither needs a guard
  float p[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) p[j] = exp_det(__fsub_rn(l[j], m));
  // the denominator: one fp32 add at a time in ascending expert order, lane
  // s extending the running sum of lanes 0 .. s-1 with its own experts (lane
  // 0 starts from 0: 0 + p_0 = p_0 exactly)
  float S = 0.f;
#pragma unroll 1
  for (int step = 0; step < 8; ++step) {
    float acc = __shfl_sync(0xffffffffu, S, gb | ((step + 7) & 7));
#pragma unroll
    for (int j = 0; j < EPL; ++j) acc = __fadd_rn(acc, p[j]);
    S = s == step ? acc : S;                   // (no branch: every lane adds, one keeps)
  }
  S = __shfl_sync(0xffffffffu, S, gb | 7);
  // p_j = RN(e_j / S), the fp32 quotient rounded once, without a division a
  // slot: with y = RN64(1 / S), RN32(RN64(e_j * y)) is that quotient whenever
  // it is a normal fp32 number.  The fp64 value is within 2^-52 (relative)
  // of e_j / S, and a normal fp32 quotient of normal operands is never
  // closer than 2^-49 to a midpoint between fp32 values (a midpoint is an odd
  // 25-bit multiple of a power of two, and e_j = S * m would then need 25
  // significant bits), so both round to the same value.  A quotient below
  // 2^-126 (e_j < S * 2^-126, e_j != 0: a logit about 87 below the
  // maximum) has fewer significant bits and can sit on a midpoint: if any
  // lane of the warp has one, the warp divides instead.
  bool tiny = false;
  const float t_min = S * 0x1p-126f;                 // exact: S >= 1
#pragma unroll
  for (int j = 0; j < EPL; ++j) tiny |= p[j] < t_min && p[j] != 0.f;
  if (__any_sync(0xffffffffu, tiny)) {
#pragma unroll
    for (int j = 0; j < EPL; ++j) p[j] = __fdiv_rn(p[j], S);
  } else {
    const double y = __drcp_rn((double)S);
#pragma unroll
    for (int j = 0; j < EPL; ++j) p[j] = __double2float_rn((double)p[j] * y);
  }
  if (live && P.probs) {
    float *pr = P.probs + t * E + e0;
    if ((E & 3) == 0) {
#pragma unroll
      for (int j = 0; j < EPL; j += 4)
        if (j < mine) *reinterpret_cast<float4 *>(pr + j) = make_float4(p[j], p[j + 1], p[j + 2], p[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (j < mine) pr[j] = p[j];
    }
  }
  if (P.topk_idx == nullptr) return;          // expert choice: probabilities only

  // ---- selection keys and gate values of the routing rule, in place --------
  //   softmax: key = logit, gate = p
  //   bias   : key = p + b_e (one fp32 add), gate = key   (DeepSeek-V3)
  //   load   : key = logit + alpha * (1 - u_e), gate = p   (load-aware top-k)
  if (P.rule != 0) {
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      if (j < mine) {
        const float st = P.state[e0 + j];
        if (P.rule == 1) {
          l[j] = __fadd_rn(p[j], st);
          p[j] = l[j];
        } else {
          l[j] = __fadd_rn(l[j], __fmul_rn(P.alpha, __fsub_rn(1.0f, st)));
        }
      }
    }
  }

  // ---- open slots: bit j set while expert e0 + j may still be chosen -------
  uint32_t open = mine >= 32 ? 0xffffffffu : ((1u << mine) - 1u);
  if (P.n_groups > 0) {
    // group g = experts [g gsz, (g+1) gsz); score = its largest key.  Lane s
    // scores groups s, s + 8, s + 16, s + 24 from the keys in shared memory.
    const int ng = P.n_groups, gsz = E / ng;
    // groups that are exactly one lane's experts (E = 8 EPL, eight groups):
    // lane s's score is its own maximum key
    const bool lane_groups = gsz == EPL && ng == 8;
    if (P.rule != 0 && !lane_groups) {
#pragma unroll
      for (int j = 0; j < EPL; j += 4)
        if (j < mine)
          *reinterpret_cast<float4 *>(lg + blk_off(r, e0 + j, NC)) = make_float4(l[j], l[j + 1], l[j + 2], l[j + 3]);
      __syncwarp();
    }
    float gsc[4];
    if (lane_groups) {
      float v = -INFINITY;
#pragma unroll
      for (int j = 0; j < EPL; ++j) v = fmaxf(v, l[j]);
      gsc[0] = v;
      gsc[1] = gsc[2] = gsc[3] = -INFINITY;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int g = s + 8 * i;
        float v = -INFINITY;
        if (g < ng)
          for (int e = g * gsz; e < g * gsz + gsz; ++e) v = fmaxf(v, lg[blk_off(r, e, NC)]);
        gsc[i] = v;
      }
    }
    uint32_t gtaken = 0, allowed = 0;
#pragma unroll 1
    for (int rr = 0; rr < P.topk_groups; ++rr) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int g = s + 8 * i;
        if (g < ng && !((gtaken >> i) & 1u) && gsc[i] > bv) {
          bv = gsc[i];
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
      if (bi < ng) {
        allowed |= 1u << bi;
        if ((bi & 7) == s) gtaken |= 1u << (bi >> 3);
      }
    }
    uint32_t amask = 0;
    for (uint32_t a = allowed; a; a &= a - 1) {
      const int g = __ffs(a) - 1;
      const int lo = max(g * gsz - e0, 0), hi = min(g * gsz + gsz - e0, mine);
      if (lo < hi) amask |= (hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u)) & ~((1u << lo) - 1u);
    }
    open &= amask;
  }

  // ---- top-k: k rounds of an arg-max over the eight lanes -------------------
  int my_idx = 0;
  float my_gate = 0.f, gsum = 0.f;
#pragma unroll 1
  for (int rr = 0; rr < k; ++rr) {
    float bv = -INFINITY, bg = 0.f;
    int bj = -1;
    // a tournament over the open slots, pairs (a, a + w) at width w = 1, 2,
    // 4, ...: the right one wins only with a strictly larger key, so the
    // lowest slot of the maximum wins (as a left-to-right scan), in log2(EPL)
    // dependent steps instead of EPL
    float tv[EPL], tg[EPL];
    int tj[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      tv[j] = ((open >> j) & 1u) != 0u ? l[j] : -INFINITY;
      tg[j] = p[j];
      tj[j] = j;
    }
#pragma unroll
    for (int w = 1; w < EPL; w <<= 1) {
#pragma unroll
      for (int a = 0; a + w < EPL; a += 2 * w) {
        const bool take = tv[a + w] > tv[a];
        tv[a] = take ? tv[a + w] : tv[a];
        tg[a] = take ? tg[a + w] : tg[a];
        tj[a] = take ? tj[a + w] : tj[a];
      }
    }
    if (tv[0] != -INFINITY) {
      bv = tv[0];
      bj = tj[0];
      bg = tg[0];
    }
    int bi = bj >= 0 ? e0 + bj : 0x7fffffff;
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
    if (bj >= 0 && bi == e0 + bj) open &= ~(1u << bj);
    if (rr == s) {
      my_idx = bi;
      my_gate = bg;
    }
    gsum = (rr == 0) ? bg : __fadd_rn(gsum, bg);
  }
  if (P.renormalize) my_gate = __fdiv_rn(my_gate, gsum);
  if (live && s < k) {
    P.topk_idx[t * k + s] = my_idx;
    P.topk_gate[t * k + s] = my_gate;
    if (hist_blk && my_idx >= 0 && my_idx < E) atomicAdd(&hist_blk[s * E + my_idx], 1);
  }
}

template <int EPL>
__global__ void __launch_bounds__(kRtThreads, 1)
    router_gate_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                          const __grid_constant__ CUtensorMap map_w, const RtParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kRtMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kRtMaxStages];
  __shared__ __align__(8) uint64_t accf_bar;
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t s_tmem_base;
  __shared__ volatile int s_abort;
  __shared__ uint64_t s_limit_sh;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ks = P.ks;
  const int c = (int)cluster_ctarank();                 // K part of this CTA
  const int64_t row0 = (int64_t)(blockIdx.x / ks) * kRtTile;
  const int TB = kRtTile / ks;                          // tokens this CTA gates
  const int64_t own0 = row0 + (int64_t)c * TB;
  const int kbc = P.K / kRtBK / ks;                     // k-blocks of a part
  const bool has_hi = row0 + 128 < P.T;                 // second 128-token half present
  const uint32_t b_bytes = (uint32_t)P.Np * kRtBK * 2;
  const uint32_t stage_bytes = 2 * kRtHalfBytes + b_bytes;
  const int NC = (P.Np + 31) / 32;                      // 32-column chunks of a row
  const size_t slot_floats = (size_t)(TB / 32) * NC * 8 * kRtBlk;
  const int nblk = TB / 32;                             // 32-token units of this CTA
  size_t region = (size_t)P.stages * stage_bytes;
  const size_t recv_bytes = (size_t)(ks - 1) * slot_floats * 4;
  if (recv_bytes > region) region = recv_bytes;
  int *s_hist = reinterpret_cast<int *>(smem + region);           // [nblk][k][E]
  const int hist_ints = P.hist ? nblk * P.k * P.E : 0;

  if (tid == 32) {
    for (int s = 0; s < P.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&accf_bar, 1);
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    tma_prefetch_map(&map_x);
    tma_prefetch_map(&map_w);
  }
  for (int i = tid; i < hist_ints; i += kRtThreads) s_hist[i] = 0;
  pdl_wait();
  pdl_trigger();
  if (tid == 0) s_limit_sh = wait_limit_ns(P.err);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  const uint64_t limit = s_limit_sh;

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------
    int stage = 0;
    uint32_t phase = 0, armed = 0, armed_parity = 0;
    bool ok = true;
    for (int i = 0; i < kbc; ++i) {
      if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort, P.err, limit)) { ok = false; break; }
      uint8_t *sa = smem + (size_t)stage * stage_bytes;
      mbar_expect_tx(&full_bar[stage], (has_hi ? 2 * kRtHalfBytes : kRtHalfBytes) + b_bytes);
      armed |= 1u << stage;
      armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
      const int kx = (c * kbc + i) * kRtBK;
      tma_load_2d(sa, &map_x, &full_bar[stage], kx, (int)row0);
      if (has_hi) tma_load_2d(sa + kRtHalfBytes, &map_x, &full_bar[stage], kx, (int)row0 + 128);
      tma_load_2d(sa + 2 * kRtHalfBytes, &map_w, &full_bar[stage], kx, 0);
      if (++stage == P.stages) { stage = 0; phase ^= 1u; }
    }
    if (!ok)
      for (int s = 0; s < P.stages; ++s)
        if (armed & (1u << s)) mbar_wait_drain(&full_bar[s], (armed_parity >> s) & 1u);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------- MMA issuer -------------------------------
    const uint32_t idesc = idesc_bf16(128, P.Np);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int i = 0; i < kbc; ++i) {
      if (!mbar_wait(&full_bar[stage], phase, &s_abort, P.err, limit)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(smem + (size_t)stage * stage_bytes);
      const uint32_t b_addr = a_addr + 2 * kRtHalfBytes;
#pragma unroll
      for (int k = 0; k < kRtBK / 16; ++k) {
        const uint64_t bd = sw128_desc(b_addr + k * 32);
        const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
        umma_bf16(tmem, sw128_desc(a_addr + k * 32), bd, idesc, acc);
        if (has_hi) umma_bf16(tmem + 256, sw128_desc(a_addr + kRtHalfBytes + k * 32), bd, idesc, acc);
      }
      umma_commit(&empty_bar[stage]);
      if (++stage == P.stages) { stage = 0; phase ^= 1u; }
    }
    if (ok) umma_commit(&accf_bar);
    umma_commit(&drain_bar);
    mbar_wait_drain(&drain_bar, 0);
  }
  __syncwarp();

  // ---- 1. accumulators complete; the cluster's stage rings are free ---------
  int okw = 1;
  if (lane == 0) okw = mbar_wait(&accf_bar, 0, &s_abort, P.err, limit) ? 1 : 0;
  okw = __shfl_sync(0xffffffffu, okw, 0);
  tc_fence_after();
  cluster_sync_all();

  // ---- 2. partial sums of the other CTAs' tokens to their receive slots -----
  // warp w reads TMEM lanes 32 (w mod 4) .. +31 of accumulator (w / 4) mod 2,
  // chunks of parity w / 8: tile rows h * 128 + 32 q + lane
  float *recv = reinterpret_cast<float *>(smem);        // [ks - 1] slots of slot_floats
  {
    const int h = (warp >> 2) & 1, q = warp & 3;
    const int tr = h * 128 + q * 32;
    const int j = tr / TB;                                // owner of these rows
    if (okw && j != c) {
      const int slot = c < j ? c : c - 1;
      const int rg = (tr - j * TB) >> 5;                  // row group in the owner's block
      const uint32_t dst0 = mapa_shared(smem_u32(recv + (size_t)slot * slot_floats), (uint32_t)j);
      for (int ch = warp >> 3; ch < NC; ch += 2) {
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t)(h * 256 + ch * 32) + ((uint32_t)(q * 32) << 16), v);
        tmem_ld_wait();
        const uint32_t dst = dst0 + (uint32_t)((((rg * NC + ch) * 8) * kRtBlk + lane * 4) * 4);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_cluster_v4(dst + (uint32_t)(i * kRtBlk * 4), v[4 * i], v[4 * i + 1], v[4 * i + 2],
                        v[4 * i + 3]);
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();

  // ---- 3. my tokens' logits: the K parts in order, then the bias ------------
  // (into receive slot 0, in place: each thread reads and writes only its
  // own row's positions)
  {
    const int q = warp & 3;
    const int hown = (c * TB) / 128, lane0 = (c * TB) & 127;
    if (okw && q * 32 >= lane0 && q * 32 < lane0 + TB) {
      const int ro = q * 32 - lane0 + lane;
      const int64_t t = own0 + ro;
      for (int ch = warp >> 2; ch < NC; ch += 4) {
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t)(hown * 256 + ch * 32) + ((uint32_t)(q * 32) << 16), v);
        tmem_ld_wait();
        const size_t base = ((size_t)((ro >> 5) * NC + ch) * 8) * kRtBlk + (ro & 31) * 4;
        float a[32];
        for (int i = 0; i < ks; ++i) {
          if (i == c) {
#pragma unroll
            for (int m = 0; m < 32; ++m)
              a[m] = (i == 0) ? __uint_as_float(v[m]) : __fadd_rn(a[m], __uint_as_float(v[m]));
          } else {
            const float *src = recv + (size_t)(i < c ? i : i - 1) * slot_floats + base;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const float4 f = *reinterpret_cast<const float4 *>(src + g * kRtBlk);
              a[4 * g] = (i == 0) ? f.x : __fadd_rn(a[4 * g], f.x);
              a[4 * g + 1] = (i == 0) ? f.y : __fadd_rn(a[4 * g + 1], f.y);
              a[4 * g + 2] = (i == 0) ? f.z : __fadd_rn(a[4 * g + 2], f.z);
              a[4 * g + 3] = (i == 0) ? f.w : __fadd_rn(a[4 * g + 3], f.w);
            }
          }
        }
        if (P.bias) {
#pragma unroll
          for (int m = 0; m < 32; ++m)
            if (ch * 32 + m < P.E) a[m] = __fadd_rn(a[m], P.bias[ch * 32 + m]);
        }
#pragma unroll
        for (int g = 0; g < 8; ++g)
          *reinterpret_cast<float4 *>(recv + base + g * kRtBlk) =
              make_float4(a[4 * g], a[4 * g + 1], a[4 * g + 2], a[4 * g + 3]);
        if (P.logits_out && t < P.T) {
          float *lo = P.logits_out + t * P.E + ch * 32;
          if ((P.E & 3) == 0 && ch * 32 + 32 <= P.E) {
#pragma unroll
            for (int m = 0; m < 32; m += 4)
              *reinterpret_cast<float4 *>(lo + m) = make_float4(a[m], a[m + 1], a[m + 2], a[m + 3]);
          } else {
#pragma unroll
            for (int m = 0; m < 32; ++m)
              if (ch * 32 + m < P.E) lo[m] = a[m];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  // ---- 4. the gate: eight lanes a token, 64 tokens a pass -------------------
  if (__all_sync(0xffffffffu, okw)) {
    const int s = tid & 7;
    for (int pass = 0; pass < TB / 64; ++pass) {
      const int tau = pass * 64 + (tid >> 3);
      const int64_t t = own0 + tau;
      int *hb = P.hist ? s_hist + (tau >> 5) * P.k * P.E : nullptr;
      gate8<EPL>(P, recv, tau, NC, t, t < P.T, s, lane, hb);
    }
  }
  if (P.y_zero) {
    const int64_t t_end = min(own0 + TB, P.T);
    const int64_t n = (t_end - own0) * P.y_vecs;
    for (int64_t i = tid; i < n; i += kRtThreads) P.y_zero[own0 * P.y_vecs + i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (P.hist) {
    __syncthreads();
    // one (block, rank) row of E counts a warp at a time, the unit number
    // once a row: group-major numbering, as the gate kernels
    for (int br = warp; br < nblk * P.k; br += kRtThreads / 32) {
      const int b = br / P.k, r = br - b * P.k;
      const int64_t B = own0 / 32 + b;                     // 32-token block
      if (B >= P.nunit) continue;
      const int64_t g = B / P.nbg, bl = B - g * P.nbg;
      int32_t *dst = P.hist + ((g * P.k + r) * P.nbg + bl) * P.E;
      const int *src = s_hist + (size_t)br * P.E;
      for (int e = lane; e < P.E; e += 32) dst[e] = src[e];
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

struct RtShape {
  int ks, Np, stages, epl;
  size_t smem;
  bool ok;
};

RtShape rt_shape(const moe_config *c) {
  RtShape r{};
  r.ok = false;
  if (c->E < 1 || c->E > kMaxExperts || c->d_model % (2 * kRtBK) != 0) return r;
  const int64_t tiles = (c->T + kRtTile - 1) / kRtTile;
  const int kb = c->d_model / kRtBK;
  // four K parts while the clusters fill one wave of SMs, else two
  r.ks = (kb % 4 == 0 && tiles * 4 <= device_sms()) ? 4 : 2;
  r.Np = (c->E + 15) / 16 * 16;
  const int TB = kRtTile / r.ks;
  const int NC = (r.Np + 31) / 32;
  const size_t recv = (size_t)(r.ks - 1) * (TB / 32) * NC * 8 * kRtBlk * 4;
  const int k = c->mode == MOE_TOKEN_CHOICE ? c->k : 0;
  const size_t hist = (size_t)(TB / 32) * k * c->E * 4;
  const size_t stage = 2 * (size_t)kRtHalfBytes + (size_t)r.Np * kRtBK * 2;
  const size_t avail = kRtSmemCap - 1024 - hist;
  int st = (int)std::min<size_t>(kRtMaxStages, avail / stage);
  if (st < 2 || recv > avail) return r;
  r.stages = st;
  const size_t region = std::max((size_t)st * stage, recv);
  // at least 120 KB: one CTA (and one 512-column TMEM allocation) an SM
  r.smem = std::max<size_t>(1024 + region + hist, 120 * 1024);
  const int epl = ((c->E + kRtLanes - 1) / kRtLanes + 3) / 4 * 4;
  r.epl = epl < 4 ? 4 : epl;
  r.ok = true;
  return r;
}

template <int EPL>
cudaError_t launch_rt(const RtShape &sh, const CUtensorMap &mx, const CUtensorMap &mw,
                      const RtParams &P, int clusters, cudaStream_t s) {
  auto kern = router_gate_tc_kernel<EPL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(clusters * sh.ks), 1, 1);
  cfg.blockDim = dim3(kRtThreads, 1, 1);
  cfg.dynamicSmemBytes = sh.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)sh.ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = MOE_PDL ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kern, mx, mw, P);
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace

bool router_tc_used(const moe_config *c) {
  return MOE_ROUTER_TC && c->dtype == MOE_BF16 && !router_is_fused(c) && rt_shape(c).ok;
}

cudaError_t launch_router_tc(const moe_config *c, const void *x, const void *w_router,
                             const float *bias, const float *state, float *logits_out, float *probs,
                             int32_t *topk_idx, float *topk_gate, int32_t *hist, void *y_zero,
                             uint32_t *err, cudaStream_t s) {
  const RtShape sh = rt_shape(c);
  if (!sh.ok) return cudaErrorInvalidValue;
  const bool tc = c->mode == MOE_TOKEN_CHOICE;
  RtParams P{};
  P.bias = bias;
  P.logits_out = logits_out;
  P.probs = probs;
  P.topk_idx = tc ? topk_idx : nullptr;
  P.topk_gate = tc ? topk_gate : nullptr;
  P.hist = tc ? hist : nullptr;
  P.state = state;
  P.rule = tc ? c->route_rule : MOE_ROUTE_SOFTMAX;
  P.alpha = c->route_alpha;
  P.T = c->T;
  P.K = c->d_model;
  P.E = c->E;
  P.Np = sh.Np;
  P.k = tc ? c->k : 0;
  P.n_groups = c->n_groups;
  P.topk_groups = c->topk_groups;
  P.renormalize = c->renormalize;
  P.nbg = unit_grid(c).nbg;
  P.nunit = (int)((c->T + kUnitTokens - 1) / kUnitTokens);
  P.ks = sh.ks;
  P.stages = sh.stages;
  P.y_zero = static_cast<uint4 *>(y_zero);
  P.y_vecs = (int)((int64_t)c->d_model * 2 / 16);
  P.err = err;
  if (tc && (P.k < 1 || P.k > kMaxTopK)) return cudaErrorInvalidValue;
  if (P.n_groups > 32) return cudaErrorInvalidValue;
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, (uint64_t)c->d_model, (uint64_t)c->T, 128)) return cudaErrorInvalidValue;
  if (!make_map(&mw, w_router, (uint64_t)c->d_model, (uint64_t)c->E, (uint32_t)sh.Np))
    return cudaErrorInvalidValue;
  const int clusters = (int)((c->T + kRtTile - 1) / kRtTile);
  switch (sh.epl) {
    case 4: return launch_rt<4>(sh, mx, mw, P, clusters, s);
    case 8: return launch_rt<8>(sh, mx, mw, P, clusters, s);
    case 12: return launch_rt<12>(sh, mx, mw, P, clusters, s);
    case 16: return launch_rt<16>(sh, mx, mw, P, clusters, s);
    case 20: return launch_rt<20>(sh, mx, mw, P, clusters, s);
    case 24: return launch_rt<24>(sh, mx, mw, P, clusters, s);
    case 28: return launch_rt<28>(sh, mx, mw, P, clusters, s);
    case 32: return launch_rt<32>(sh, mx, mw, P, clusters, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
