// Selection under capacity / keep-fraction / expert choice, and the
// permutation of kept (token, expert) pairs into expert-contiguous rows.
//
// Token choice (GShard section 1 of "MoE技术演进": expert capacity C = O(N/E),
// overflow passes through the residual): a stable counting sort of the
// assignments by expert, in priority order q = j*T + t (every first choice
// before any second choice, lower token first), in units of 32 tokens:
//   hist_units    per-unit expert histogram (the gate kernel writes it when
//                 it runs first, so moe_forward skips this launch)
//   unit_sums     per-expert totals of each block of 32 units (skipped for
//                 small histograms without local groups: the rank kernel's
//                 blocks then sum all units before theirs themselves)
//   rank_units    per block: bases from the earlier blocks' totals and an
//                 in-block scan, counts / kept rows (min(n_e, C) or
//                 ceil(n_e*num/den)) / row offsets; then the stable rank of
//                 each assignment inside its expert (warp match within the
//                 unit), the capacity test and the slot / row writes -- or,
//                 for keep-fraction, the expert-grouped list
//   keep_select   per expert, the ceil(n_e*num/den) assignments with the
//                 largest p[t, e] (DeepSeek-V2 section 5, token dropping)
// Expert choice (LocMoE+ article: each expert picks its top-C tokens):
//   transpose     probs [T, E] -> [E, T]
//   ec_select     per expert, the C tokens with the largest p[t, e], rows in
//                 ascending t
// Both selections use an exact radix select over the 64-bit key
// (p bits << 32 | ~t), so "larger p first, lower t on ties" is decided by
// integer comparisons alone.
//   scatter_rows  x_perm[r] = x[row_token[r]], written token by token: one
//                 warp per token reads its row of x once and writes it to
//                 each of its rows (16-byte vectors).  (gather_rows, one
//                 warp per row, is the build-time alternative.)
#include <algorithm>
#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

// ---------------------------------------------------------------------------
// row gather: x_perm[r] = x[row_token[r]] for r < offsets[E], one warp per
// row (grid-stride), 16-byte vectors, four loads in flight per lane.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ x,
                                                          uint4 *__restrict__ x_perm,
                                                          const int32_t *__restrict__ row_token,
                                                          const int32_t *__restrict__ offsets, int E,
                                                          int64_t T, int vpr, uint32_t *err) {
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  const int64_t R = offsets[E];
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += nwarps) {
    const int64_t t = row_token[r];
    if (t < 0 || t >= T) {
      if (lane == 0) raise_error(err, kErrBadIndex);
      continue;
    }
    const uint4 *src = x + t * vpr;
    uint4 *dst = x_perm + r * vpr;
    int v = lane;
    for (; v + 96 < vpr; v += 128) {
      const uint4 a = src[v], b = src[v + 32], c = src[v + 64], d = src[v + 96];
      dst[v] = a;
      dst[v + 32] = b;
      dst[v + 64] = c;
      dst[v + 96] = d;
    }
    for (; v < vpr; v += 32) dst[v] = src[v];
  }
}

// ---------------------------------------------------------------------------
// The same rows written token by token.  One warp per token collects the
// rows of its kept choices (token choice: tok_rows[t * k + j]; expert
// choice: tok_rows[e * T + t] over the experts; -1: not kept), then reads
// x[t] once, 8 16-byte vectors a lane at a time, and writes each piece to
// every one of those rows.  Every row of x crosses HBM once; the row-by-row
// gather above re-reads a token's row for each of its rows, and the repeats
// mostly miss L2 while the x_perm writes stream through it.
// ---------------------------------------------------------------------------
#ifndef MOE_SCATTER
#define MOE_SCATTER 1
#endif
constexpr int kScatterWarps = 8;
__global__ void __launch_bounds__(kScatterWarps * 32) scatter_rows_kernel(
    const uint4 *__restrict__ x, uint4 *__restrict__ x_perm, const int32_t *__restrict__ tok_rows,
    int64_t T, int W, int expert_major, int vpr, int64_t rows_cap, uint32_t *err) {
  __shared__ int s_rows[kScatterWarps][kMaxExperts];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int *rows = s_rows[warp];
  pdl_wait();
  pdl_trigger();
  const int64_t nwarps = (int64_t)gridDim.x * kScatterWarps;
  for (int64_t t = (int64_t)blockIdx.x * kScatterWarps + warp; t < T; t += nwarps) {
    int n = 0;
    for (int c = 0; c < W; c += 32) {
      const int w = c + lane;
      int r = -1;
      if (w < W) {
        r = expert_major ? tok_rows[(int64_t)w * T + t] : tok_rows[t * W + w];
        if (r >= rows_cap) {
          raise_error(err, kErrBadIndex);
          r = -1;
        }
      }
      const unsigned valid = __ballot_sync(0xffffffffu, r >= 0);
      if (r >= 0) rows[n + __popc(valid & ((1u << lane) - 1u))] = r;
      n += __popc(valid);
    }
    __syncwarp();
    const uint4 *src = x + t * vpr;
    for (int v0 = 0; v0 < vpr; v0 += 32 * 8) {
      uint4 buf[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < vpr) buf[i] = src[v];
      }
      for (int j = 0; j < n; ++j) {
        uint4 *dst = x_perm + (int64_t)rows[j] * vpr;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int v = v0 + i * 32 + lane;
          if (v < vpr) dst[v] = buf[i];
        }
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// token choice: histogram of the priority order, per 32-token unit.
// Unit u = r * nunit + b covers the rank-r choices of tokens b*32 .. b*32+31,
// i.e. priorities q = r*T + b*32 + lane: units in index order are the
// priority order.  (When the gate runs first it writes this histogram
// itself; this kernel serves moe_permute called on its own.)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hist_units_kernel(const int32_t *__restrict__ topk_idx,
                                                         int64_t T, int k, int E, int nu, int nbg,
                                                         int32_t *__restrict__ hist, uint32_t *err) {
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  const int64_t u = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (u >= nu) return;                                   // whole warp leaves together
  // unit u = g*k*nbg + r*nbg + bl (local groups; one group: g = 0)
  const int64_t g = u / ((int64_t)k * nbg);
  const int64_t rem = u - g * k * nbg;
  const int r = (int)(rem / nbg);
  const int64_t b = g * nbg + (rem - (int64_t)r * nbg);
  const int64_t t = b * kUnitTokens + lane;
  int e = -1;
  if (t < T) {
    e = topk_idx[t * k + r];
    if (e < 0 || e >= E) {
      raise_error(err, kErrBadIndex);
      e = -1;
    }
  }
  int32_t *h = hist + u * E;
  for (int i = lane; i < E; i += 32) h[i] = 0;
  __syncwarp();
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  if (e >= 0 && (__ffs(peers) - 1) == lane) h[e] = __popc(peers);
}

// ---------------------------------------------------------------------------
// token choice: scans, in two levels.  Units are grouped in blocks of
// kUnitsPerBlock; unit_sums gives each block's per-expert total; the rank
// kernel of a block then adds up the totals of the blocks before it, scans
// its own units in shared memory, and has the per-expert base of each unit.
// Every block also derives counts, kept rows (min(n_e, C) or
// ceil(n_e*num/den)) and the exclusive scans over experts from the totals;
// block 0 writes them out.
// ---------------------------------------------------------------------------

// units of scan block b: kUnitsPerBlock consecutive units of one local group
__device__ __forceinline__ void block_units(int b, int upg, int bpg, int &u_begin, int &u_end) {
  const int g = b / bpg;
  u_begin = g * upg + (b - g * bpg) * kUnitsPerBlock;
  u_end = min(u_begin + kUnitsPerBlock, (g + 1) * upg);
}

__global__ void __launch_bounds__(1024) unit_sums_kernel(const int32_t *__restrict__ hist, int upg,
                                                         int bpg, int E, int32_t *__restrict__ bsum) {
  __shared__ int s_part[1024];
  pdl_wait();
  pdl_trigger();
  const int G = max(1, (int)blockDim.x / E);
  const int g = threadIdx.x / E, e = threadIdx.x - g * E;
  int u_begin, u_end;
  block_units(blockIdx.x, upg, bpg, u_begin, u_end);
  int part = 0;
  if (g < G)
    for (int u = u_begin + g; u < u_end; u += G) part += hist[(int64_t)u * E + e];
  if (g < G) s_part[threadIdx.x] = part;
  __syncthreads();
  if (g == 0) {
    int total = 0;
    for (int gg = 0; gg < G; ++gg) total += s_part[gg * E + e];
    bsum[(int64_t)blockIdx.x * E + e] = total;
  }
}

// ---------------------------------------------------------------------------
// token choice: stable rank of each assignment inside its expert.  Block b
// owns units b*32 .. b*32+31, one warp per unit: rank = per-expert base of
// the unit + rank among equal experts inside the unit (warp match).  Then the
// capacity test and the slot / row writes -- or, for keep-fraction, the
// expert-grouped list of priorities.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024, 1) rank_units_kernel(
    const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_gate, int64_t T, int k,
    int E, int nbg, int upg, int bpg, int nb, const int32_t *__restrict__ hist,
    const int32_t *__restrict__ bsum, int capacity, int keep_num, int keep_den, int keep_fraction,
    int32_t *__restrict__ counts,
    int32_t *__restrict__ cnt_off_out, int32_t *__restrict__ kept_out,
    int32_t *__restrict__ offsets_out, int32_t *__restrict__ n_dropped,
    int32_t *__restrict__ tok_rows, int32_t *__restrict__ row_token, float *__restrict__ row_gate,
    int32_t *__restrict__ sorted_q) {
  extern __shared__ int sm[];
  pdl_wait();
  pdl_trigger();
  int *s_base = sm;                                   // [32 units][E]
  int *s_pre = s_base + kUnitsPerBlock * E;           // [E] totals of earlier blocks
  int *s_tot = s_pre + E;                             // [E] totals of all blocks
  int *s_off = s_tot + E;                             // [E+1] row offsets (exclusive scan of kept)
  int *s_coff = s_off + E + 1;                        // [E+1] count offsets
  int *s_part = s_coff + E + 1;                       // [1024] partial sums
  int *s_part2 = s_part + 1024;                       // [1024]
  int *s_kept = s_part2 + 1024;                       // [E] rows kept (local groups)
  int *s_kbefore = s_kept + E;                        // [E] rows kept by earlier groups
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  int u_begin, u_end;
  block_units(b, upg, bpg, u_begin, u_end);
  const int lgroups = nb / bpg;                       // local groups
  const int my_group = b / bpg;

  // this warp's unit (u = g*upg + r*nbg + bl) and its lane's assignment,
  // loaded now so that the loads overlap the scans below
  const int u = u_begin + warp;
  const bool unit_live = u < u_end;
  int r = 0, e = -1;
  int64_t t = 0;
  float gate = 0.f;
  if (unit_live) {
    const int rem = u - my_group * upg;
    r = rem / nbg;
    const int64_t bu = (int64_t)my_group * nbg + (rem - r * nbg);
    t = bu * kUnitTokens + lane;
    if (t < T) {
      e = topk_idx[t * k + r];
      if (e < 0 || e >= E) e = -1;                       // reported by the histogram
      if (!keep_fraction && e >= 0) gate = topk_gate[t * k + r];
    }
  }

  // 1. totals of the blocks before this one (in its group), and of all blocks
  const int G = max(1, (int)blockDim.x / E);
  const int g = threadIdx.x / E, e_g = threadIdx.x - g * E;
  if (lgroups == 1 && bsum == nullptr) {
    // small histograms: every block sums the units itself (no unit_sums launch)
    int pre = 0, tot = 0;
    if (g < G) {
      for (int u = g; u < upg; u += G) {
        const int v = hist[(int64_t)u * E + e_g];
        tot += v;
        if (u < u_begin) pre += v;
      }
      s_part[threadIdx.x] = pre;
      s_part2[threadIdx.x] = tot;
    }
  } else if (lgroups == 1) {
    int pre = 0, tot = 0;
    if (g < G) {
      for (int bb = g; bb < nb; bb += G) {
        const int v = bsum[(int64_t)bb * E + e_g];
        tot += v;
        if (bb < b) pre += v;
      }
      s_part[threadIdx.x] = pre;
      s_part2[threadIdx.x] = tot;
    }
  } else {
    // local groups: per expert, one thread walks every group's blocks
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int pre = 0, tot = 0, kept = 0, kbefore = 0;
      for (int gg = 0; gg < lgroups; ++gg) {
        int n = 0;
        for (int bb = gg * bpg; bb < (gg + 1) * bpg; ++bb) {
          const int v = bsum[(int64_t)bb * E + e];
          n += v;
          if (gg == my_group && bb < b) pre += v;
        }
        const int kg = capacity > 0 ? min(n, capacity) : n;
        tot += n;
        kept += kg;
        if (gg < my_group) kbefore += kg;
      }
      s_pre[e] = pre;
      s_tot[e] = tot;
      s_kept[e] = kept;
      s_kbefore[e] = kbefore;
    }
  }
  // this block's unit histograms into shared memory
  for (int i = threadIdx.x; i < (u_end - u_begin) * E; i += blockDim.x)
    s_base[i] = hist[(int64_t)u_begin * E + i];
  __syncthreads();
  if (lgroups == 1 && g == 0) {
    int p = 0, t = 0;
    for (int gg = 0; gg < G; ++gg) {
      p += s_part[gg * E + e_g];
      t += s_part2[gg * E + e_g];
    }
    s_pre[e_g] = p;
    s_tot[e_g] = t;
    s_kbefore[e_g] = 0;
  }
  __syncthreads();
  // 2. per-expert exclusive scan over this block's units (in place)
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = s_pre[e];
    for (int i = 0; i < u_end - u_begin; ++i) {
      const int v = s_base[i * E + e];
      s_base[i * E + e] = run;
      run += v;
    }
  }
  // 3. kept rows and the exclusive scans over experts
  if (warp == 0) {
    int a = 0, c = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int ce = e < E ? s_tot[e] : 0;
      int ke = ce;
      if (lgroups > 1) ke = e < E ? s_kept[e] : 0;
      else if (capacity > 0) ke = min(ce, capacity);
      else if (keep_den > 0) ke = (int)(((int64_t)ce * keep_num + keep_den - 1) / keep_den);
      int xa = ce, xc = ke;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, xa, o);
        const int yc = __shfl_up_sync(0xffffffffu, xc, o);
        if (lane >= o) {
          xa += ya;
          xc += yc;
        }
      }
      if (e < E) {
        s_coff[e] = a + xa - ce;
        s_off[e] = c + xc - ke;
        if (b == 0) {
          counts[e] = ce;
          kept_out[e] = ke;
          cnt_off_out[e] = a + xa - ce;
          offsets_out[e] = c + xc - ke;
        }
      }
      a += __shfl_sync(0xffffffffu, xa, 31);
      c += __shfl_sync(0xffffffffu, xc, 31);
    }
    if (lane == 0) {
      s_coff[E] = a;
      s_off[E] = c;
      if (b == 0) {
        cnt_off_out[E] = a;
        offsets_out[E] = c;
        *n_dropped = (int)((int64_t)T * k - c);
      }
    }
  }
  __syncthreads();

  // 4. one warp per unit: the rank of each assignment inside its expert
  if (!unit_live) return;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = e >= 0 ? s_base[warp * E + e] + __popc(peers & ((1u << lane) - 1u)) : 0;
  if (keep_fraction) {
    if (e >= 0) sorted_q[s_coff[e] + rank] = (int32_t)(r * T + t);
    return;
  }
  const bool keep = e >= 0 && (capacity <= 0 || rank < capacity);
  const int slot = keep ? s_off[e] + s_kbefore[e] + rank : -1;
  if (e >= 0) tok_rows[t * k + r] = slot;
  if (keep) {
    row_token[slot] = (int32_t)t;
    row_gate[slot] = gate;
  }
}

// ---------------------------------------------------------------------------
// block helpers (1024 threads)
// ---------------------------------------------------------------------------
// Exclusive scan of one int per thread over the whole block; *total receives
// the block sum.  Ends with a barrier, so `scratch` may be reused at once.
__device__ __forceinline__ int block_exclusive_scan(int v, int *scratch, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    scratch[lane] = w;
  }
  __syncthreads();
  const int before = warp > 0 ? scratch[warp - 1] : 0;
  *total = scratch[nwarps - 1];
  __syncthreads();
  return before + x - v;
}

// The m-th largest (1-based) of n distinct 64-bit keys, keys produced by
// key_of(i) for i in [0, n).  Exact radix select, 8 bits per pass, MSB first.
template <class KeyOf>
__device__ uint64_t block_select_kth_largest(int n, int m, KeyOf key_of, int *hist /*[256]*/,
                                             uint64_t *s_prefix, int *s_remaining) {
  if (threadIdx.x == 0) {
    *s_prefix = 0ull;
    *s_remaining = m;
  }
  __syncthreads();
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    const uint64_t hm = (pass == 0) ? 0ull : (~0ull << (shift + 8));
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint64_t prefix = *s_prefix;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint64_t key = key_of(i);
      if ((key & hm) == (prefix & hm)) atomicAdd(&hist[(key >> shift) & 0xff], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int remaining = *s_remaining, acc = 0, digit = 0;
      for (int d = 255; d >= 0; --d) {
        if (acc + hist[d] >= remaining) { digit = d; break; }
        acc += hist[d];
      }
      *s_remaining = remaining - acc;
      *s_prefix = prefix | ((uint64_t)digit << shift);
    }
    __syncthreads();
  }
  return *s_prefix;
}

// ---------------------------------------------------------------------------
// token choice, keep-fraction: per-expert affinity selection
// ---------------------------------------------------------------------------
// lists of at most this many assignments select by counting (n^2 / 1024
// compares a thread) instead of the 8-pass radix select
constexpr int kKeepCountMax = 2048;

__global__ void __launch_bounds__(1024) keep_select_kernel(
    const int32_t *__restrict__ sorted_q, const int32_t *__restrict__ cnt_off,
    const int32_t *__restrict__ kept, const int32_t *__restrict__ offsets,
    const float *__restrict__ probs, const float *__restrict__ topk_gate, int64_t T, int k, int E,
    int32_t *__restrict__ tok_rows, int32_t *__restrict__ row_token, float *__restrict__ row_gate) {
  __shared__ int hist[256];
  __shared__ int scratch[32];
  __shared__ uint64_t s_prefix;
  __shared__ int s_remaining;
  __shared__ uint64_t s_keys[kKeepCountMax];
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  const int start = cnt_off[e];
  const int n = cnt_off[e + 1] - start;
  const int m = kept[e];
  const int32_t *list = sorted_q + start;
  // q = j * T + t < T * k <= 2^31 - 1 (validated): 32-bit division is exact
  const uint32_t T32 = (uint32_t)T;
  auto key_of = [&](int i) -> uint64_t {
    const uint32_t t = (uint32_t)list[i] % T32;
    return affinity_key(probs[(int64_t)t * E + e], t);
  };
  uint64_t thr = 0ull;          // keep keys >= thr
  bool keep_all = m >= n, keep_none = m <= 0;
  if (!keep_all && !keep_none) {
    if (n <= kKeepCountMax) {
      // short lists: the m-th largest key by counting, for each key, the keys
      // above it (keys are distinct: each token appears once in a list); the
      // key with exactly m - 1 above it is the threshold
      for (int i = threadIdx.x; i < n; i += blockDim.x) s_keys[i] = key_of(i);
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const uint64_t ki = s_keys[i];
        int above = 0;
        for (int j = 0; j < n; ++j) above += s_keys[j] > ki ? 1 : 0;
        if (above == m - 1) s_prefix = ki;
      }
      __syncthreads();
      thr = s_prefix;
    } else {
      thr = block_select_kth_largest(n, m, key_of, hist, &s_prefix, &s_remaining);
    }
  }
  const int row0 = offsets[e];
  int done = 0;
  for (int c = 0; c < n; c += blockDim.x) {
    const int i = c + threadIdx.x;
    bool keep = false;
    int64_t q = 0;
    if (i < n) {
      q = list[i];
      keep = keep_all || (!keep_none && key_of(i) >= thr);
    }
    int total;
    const int r = block_exclusive_scan(keep ? 1 : 0, scratch, &total);
    if (i < n) {
      const int64_t j = (uint32_t)q / T32, t = q - j * T;
      if (keep) {
        const int slot = row0 + done + r;
        tok_rows[t * k + j] = slot;
        row_token[slot] = (int32_t)t;
        row_gate[slot] = topk_gate[t * k + j];
      } else {
        tok_rows[t * k + j] = -1;
      }
    }
    done += total;
  }
}

// ---------------------------------------------------------------------------
// expert choice
// ---------------------------------------------------------------------------
__global__ void transpose_kernel(const float *__restrict__ in, float *__restrict__ out, int64_t T,
                                 int E) {
  __shared__ float tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int e0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t t = t0 + i;
    const int e = e0 + threadIdx.x;
    if (t < T && e < E) tile[i][threadIdx.x] = in[t * E + e];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int e = e0 + i;
    const int64_t t = t0 + threadIdx.x;
    if (t < T && e < E) out[(int64_t)e * T + t] = tile[threadIdx.x][i];
  }
}

__global__ void __launch_bounds__(1024) ec_select_kernel(
    const float *__restrict__ probs_t, int64_t T, int E, int C, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ tok_rows, int32_t *__restrict__ row_token,
    float *__restrict__ row_gate, int32_t *__restrict__ n_dropped) {
  __shared__ int hist[256];
  __shared__ int scratch[32];
  __shared__ uint64_t s_prefix;
  __shared__ int s_remaining;
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  const float *pe = probs_t + (int64_t)e * T;
  auto key_of = [&](int i) -> uint64_t { return affinity_key(pe[i], (uint32_t)i); };
  const int n = (int)T;
  const bool keep_all = C >= n;
  uint64_t thr = 0ull;
  if (!keep_all) thr = block_select_kth_largest(n, C, key_of, hist, &s_prefix, &s_remaining);
  if (threadIdx.x == 0) {
    counts[e] = C;
    offsets[e] = e * C;
    if (e == E - 1) {
      offsets[E] = E * C;
      *n_dropped = 0;
    }
  }
  int done = 0;
  for (int c = 0; c < n; c += blockDim.x) {
    const int t = c + threadIdx.x;
    bool keep = false;
    if (t < n) keep = keep_all || key_of(t) >= thr;
    int total;
    const int r = block_exclusive_scan(keep ? 1 : 0, scratch, &total);
    if (t < n) {
      if (keep) {
        const int row = e * C + done + r;
        tok_rows[(int64_t)e * T + t] = row;
        row_token[row] = t;
        row_gate[row] = pe[t];
      } else {
        tok_rows[(int64_t)e * T + t] = -1;
      }
    }
    done += total;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
cudaError_t launch_permute(const moe_config *c, const WsLayout &L, char *ws, bool hist_ready,
                           const void *x, const int32_t *topk_idx, const float *topk_gate,
                           const float *probs, int32_t *counts, int32_t *offsets, int32_t *tok_rows,
                           int32_t *row_token, float *row_gate, void *x_perm, int32_t *n_dropped,
                           cudaStream_t s, bool gather) {
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + L.err);
  const int E = c->E;
  const int64_t T = c->T;
  const int vpr = (int)(c->d_model * elem_size(c) / 16);
  const uint4 *xv = reinterpret_cast<const uint4 *>(x);
  uint4 *xp = reinterpret_cast<uint4 *>(x_perm);
  if (c->mode == MOE_EXPERT_CHOICE) {
    float *pt = reinterpret_cast<float *>(ws + L.probs_t);
    dim3 tb(32, 8), tg((unsigned)((T + 31) / 32), (unsigned)((E + 31) / 32));
    cudaError_t e = launch_kernel(transpose_kernel, tg, tb, 0, s, probs, pt, T, E);
    if (e != cudaSuccess) return e;
    e = launch_kernel(ec_select_kernel, E, 1024, 0, s, pt, T, E, c->ec_capacity, counts, offsets,
                      tok_rows, row_token, row_gate, n_dropped);
    if (e != cudaSuccess) return e;
  } else {
  int32_t *hist = reinterpret_cast<int32_t *>(ws + L.hist);
  int32_t *bsum = reinterpret_cast<int32_t *>(ws + L.base);
  int32_t *cnt_off = reinterpret_cast<int32_t *>(ws + L.cnt_off);
  int32_t *kept = reinterpret_cast<int32_t *>(ws + L.kept);
  int32_t *sorted_q = reinterpret_cast<int32_t *>(ws + L.sorted_q);
  const int capacity = (int)capacity_rows(c);                // 0: unlimited
  const int keepfrac = (capacity == 0 && c->keep_den > 0) ? 1 : 0;
  const UnitGrid ug = unit_grid(c);
  const int nu = ug.G * ug.upg;
  const int nb = ug.nb;
  cudaError_t e = cudaSuccess;
  if (!hist_ready) {
    e = launch_kernel(hist_units_kernel, (unsigned)((nu + 7) / 8), 256, 0, s, topk_idx, T, c->k, E,
                      nu, ug.nbg, hist, err);
    if (e != cudaSuccess) return e;
  }
  // without local groups and with at most 16K histogram entries, the rank
  // kernel's blocks sum the units before them themselves (one launch fewer)
  const bool own_sums = ug.G == 1 && (int64_t)nu * E <= 16384;
  if (!own_sums) {
    e = launch_kernel(unit_sums_kernel, nb, 1024, 0, s, hist, ug.upg, ug.bpg, E, bsum);
    if (e != cudaSuccess) return e;
  }
  const size_t rank_smem = ((size_t)kUnitsPerBlock * E + 6 * E + 2 + 2048) * sizeof(int);
  if (rank_smem > 48 * 1024) {
    e = cudaFuncSetAttribute(rank_units_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)rank_smem);
    if (e != cudaSuccess) return e;
  }
  e = launch_kernel(rank_units_kernel, nb, 1024, rank_smem, s, topk_idx, topk_gate, T, c->k, E,
                    ug.nbg, ug.upg, ug.bpg, nb, hist, own_sums ? nullptr : bsum, capacity,
                    c->keep_num, c->keep_den,
                    keepfrac, counts,
                    cnt_off, kept, offsets, n_dropped, tok_rows, row_token, row_gate, sorted_q);
  if (e != cudaSuccess) return e;
  if (keepfrac) {
    e = launch_kernel(keep_select_kernel, E, 1024, 0, s, sorted_q, cnt_off, kept, offsets, probs,
                      topk_gate, T, c->k, E, tok_rows, row_token, row_gate);
    if (e != cudaSuccess) return e;
  }
  }
  if (!gather) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (MOE_SCATTER) {
    const bool ec = c->mode == MOE_EXPERT_CHOICE;
    const int64_t tw = (T + kScatterWarps - 1) / kScatterWarps;
    const int tblocks = (int)std::max<int64_t>(1, std::min<int64_t>(tw, (int64_t)sms * 8));
    return launch_kernel(scatter_rows_kernel, tblocks, kScatterWarps * 32, 0, s, xv, xp,
                         static_cast<const int32_t *>(tok_rows), T, ec ? E : c->k, ec ? 1 : 0, vpr,
                         L.rows_cap, err);
  }
  const int64_t want = (L.rows_cap + 7) / 8;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
  return launch_kernel(gather_rows_kernel, blocks, 256, 0, s, xv, xp, row_token, offsets, E, T, vpr,
                       err);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_permute_noalloc: moe_permute for callers that cannot allocate.
//
// Some callers cannot allocate device memory at all: a plugin inside a host
// program that hands it only its input and output buffers, or a process that
// must keep a fixed device footprint once it has started.  They cannot
// provide moe_permute's workspace.  This entry point takes its scratch from
// one fixed array compiled into the library instead.
//
// The array lives on every GPU that loads the library until the process
// exits.  In host code its name is only a host-side stand-in, so its device
// address is looked up (with the device current) through
// cudaGetSymbolAddress and passed to the kernels like a workspace pointer.
// Only the permutation's share of a workspace (control block, histograms,
// scans, keep-fraction list or transposed probabilities) lives there.
// All calls on a device share the array and it keeps the last call's
// contents: the kernels overwrite every scratch word they read except the
// error word, which each call clears first.  Calls that overlap on the GPU
// race on the array.
// ---------------------------------------------------------------------------
namespace moe {

constexpr size_t kStaticScratchBytes = MOE_PERMUTE_NOALLOC_SCRATCH_BYTES;     // 8 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_address[kMaxDevices] = {};

// Device address of g_static_scratch on the current device.  Looked up
// again on every call whose stream is not capturing (cheap; a device reset
// reloads the module and can move the array), the cached address reused
// while the stream captures (a lookup may not be legal then).
cudaError_t static_scratch_address(cudaStream_t s, char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (cap == cudaStreamCaptureStatusNone || g_scratch_address[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_address[dev] = p;
  }
  *out = static_cast<char *>(g_scratch_address[dev]);
  return cudaSuccess;
}
}  // namespace

}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_config *cfg, const void *x,
                                          const int32_t *topk_idx, const float *topk_gate,
                                          const float *probs, int32_t *counts, int32_t *offsets,
                                          int32_t *tok_rows, int32_t *row_token, float *row_gate,
                                          void *x_perm, int32_t *n_dropped, moe_stream_t stream) {
  using namespace moe;
  const moe_status st = validate(cfg);
  if (st != MOE_OK) return st;
  const WsLayout L = make_layout(cfg);
  // the permutation's scratch (moe_sizes.permute_workspace) must fit the array
  if (L.permute_end > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  const bool tc = cfg->mode == MOE_TOKEN_CHOICE;
  const bool keepfrac = tc && capacity_rows(cfg) == 0 && cfg->keep_den > 0;
  if (!x || !counts || !offsets || !tok_rows || !row_token || !row_gate || !x_perm || !n_dropped)
    return MOE_ERR_INVALID_ARG;
  if (tc && (!topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if ((!tc || keepfrac) && !probs) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *scratch = nullptr;
  if (static_scratch_address(s, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemsetAsync(scratch + L.err, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e = launch_permute(cfg, L, scratch, false, x, topk_idx, topk_gate, probs, counts,
                                       offsets, tok_rows, row_token, row_gate, x_perm, n_dropped, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
