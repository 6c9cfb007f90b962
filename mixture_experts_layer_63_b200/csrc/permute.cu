// Selection under capacity / keep-fraction / expert choice, and the
// permutation of kept (token, expert) pairs into expert-contiguous rows.
//
// Token choice (GShard section 1 of "MoE技术演进": expert capacity C = O(N/E),
// overflow passes through the residual): a stable counting sort of the
// assignments by expert, in priority order q = j*T + t (every first choice
// before any second choice, lower token first):
//   hist_kernel   per-block expert histogram over q
//   scan_kernel   per-expert exclusive scan over blocks, counts, kept rows
//                 (min(n_e, C), or ceil(n_e*num/den)) and row offsets
//   rank_kernel   stable rank of each assignment inside its expert (warp
//                 match + per-warp prefix), then the capacity test and the
//                 slot / row writes -- or, for keep-fraction, the grouped list
//   keep_select   per expert, the ceil(n_e*num/den) assignments with the
//                 largest p[t, e] (DeepSeek-V2 section 5, token dropping)
// Expert choice (LocMoE+ article: each expert picks its top-C tokens):
//   transpose     probs [T, E] -> [E, T]
//   ec_select     per expert, the C tokens with the largest p[t, e], rows in
//                 ascending t
// Both selections use an exact radix select over the 64-bit key
// (p bits << 32 | ~t), so "larger p first, lower t on ties" is decided by
// integer comparisons alone.
//   gather_rows   x_perm[r] = x[row_token[r]], 16-byte vectors.
#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

// ---------------------------------------------------------------------------
// token choice: histogram
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) hist_kernel(const int32_t *__restrict__ topk_idx, int64_t T,
                                                   int k, int E, int32_t *__restrict__ hist,
                                                   uint32_t *err) {
  __shared__ int h[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int64_t Q = T * k;
  const int64_t q0 = (int64_t)blockIdx.x * kAssignBlock;
  const int64_t q1 = min(q0 + kAssignBlock, Q);
  for (int64_t q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
    const int64_t j = q / T, t = q - j * T;
    const int e = topk_idx[t * k + j];
    if (e < 0 || e >= E) { raise_error(err, kErrBadIndex); continue; }
    atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)blockIdx.x * E + e] = h[e];
}

// ---------------------------------------------------------------------------
// token choice: scans
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) scan_kernel(const int32_t *__restrict__ hist, int nblk, int E,
                                                   int64_t Q, int capacity, int keep_num,
                                                   int keep_den, int32_t *__restrict__ base,
                                                   int32_t *__restrict__ counts,
                                                   int32_t *__restrict__ cnt_off,
                                                   int32_t *__restrict__ kept,
                                                   int32_t *__restrict__ offsets,
                                                   int32_t *__restrict__ n_dropped) {
  __shared__ int s_cnt[kMaxExperts];
  __shared__ int s_kept[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int b = 0; b < nblk; ++b) {
      base[(int64_t)b * E + e] = run;
      run += hist[(int64_t)b * E + e];
    }
    int kp = run;
    if (capacity > 0) kp = min(run, capacity);
    else if (keep_den > 0) kp = (int)(((int64_t)run * keep_num + keep_den - 1) / keep_den);
    s_cnt[e] = run;
    s_kept[e] = kp;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int e = 0; e < E; ++e) {
      cnt_off[e] = a;
      offsets[e] = b;
      counts[e] = s_cnt[e];
      kept[e] = s_kept[e];
      a += s_cnt[e];
      b += s_kept[e];
    }
    cnt_off[E] = a;
    offsets[E] = b;
    *n_dropped = (int)(Q - b);
  }
}

// ---------------------------------------------------------------------------
// token choice: stable rank inside the expert, then slot / row writes
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rank_kernel(
    const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_gate, int64_t T, int k,
    int E, const int32_t *__restrict__ base, const int32_t *__restrict__ offsets,
    const int32_t *__restrict__ cnt_off, int capacity, int keep_fraction,
    int32_t *__restrict__ tok_rows, int32_t *__restrict__ row_token, float *__restrict__ row_gate,
    int32_t *__restrict__ sorted_q) {
  __shared__ int running[kMaxExperts];
  __shared__ int wc[8][kMaxExperts];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    running[e] = base[(int64_t)blockIdx.x * E + e];
#pragma unroll
    for (int w = 0; w < 8; ++w) wc[w][e] = 0;
  }
  __syncthreads();
  const int64_t Q = T * k;
  const int64_t q0 = (int64_t)blockIdx.x * kAssignBlock;
  const int64_t q1 = min(q0 + kAssignBlock, Q);
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int64_t cq = q0; cq < q1; cq += blockDim.x) {
    const int64_t q = cq + threadIdx.x;
    int e = -1;
    int64_t t = 0, j = 0;
    if (q < q1) {
      j = q / T;
      t = q - j * T;
      e = topk_idx[t * k + j];
      if (e < 0 || e >= E) e = -1;       // reported by hist_kernel
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int lane_rank = __popc(peers & lt_mask);
    const int cnt = __popc(peers);
    const bool leader = (__ffs(peers) - 1) == lane;
    if (e >= 0 && leader) wc[warp][e] = cnt;
    __syncthreads();
    int rank = 0;
    if (e >= 0) {
      rank = running[e] + lane_rank;
      for (int w = 0; w < warp; ++w) rank += wc[w][e];
    }
    __syncthreads();
    if (e >= 0 && leader) {
      atomicAdd(&running[e], cnt);      // leaders of several warps may share e
      wc[warp][e] = 0;
    }
    __syncthreads();
    if (e < 0) continue;
    if (keep_fraction) {
      sorted_q[cnt_off[e] + rank] = (int32_t)q;
    } else {
      const bool keep = capacity <= 0 || rank < capacity;
      const int slot = keep ? offsets[e] + rank : -1;
      tok_rows[t * k + j] = slot;
      if (keep) {
        row_token[slot] = (int32_t)t;
        row_gate[slot] = topk_gate[t * k + j];
      }
    }
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
__global__ void __launch_bounds__(1024) keep_select_kernel(
    const int32_t *__restrict__ sorted_q, const int32_t *__restrict__ cnt_off,
    const int32_t *__restrict__ kept, const int32_t *__restrict__ offsets,
    const float *__restrict__ probs, const float *__restrict__ topk_gate, int64_t T, int k, int E,
    int32_t *__restrict__ tok_rows, int32_t *__restrict__ row_token, float *__restrict__ row_gate) {
  __shared__ int hist[256];
  __shared__ int scratch[32];
  __shared__ uint64_t s_prefix;
  __shared__ int s_remaining;
  const int e = blockIdx.x;
  const int start = cnt_off[e];
  const int n = cnt_off[e + 1] - start;
  const int m = kept[e];
  const int32_t *list = sorted_q + start;
  auto key_of = [&](int i) -> uint64_t {
    const int64_t q = list[i];
    const int64_t t = q % T;
    return affinity_key(probs[t * E + e], (uint32_t)t);
  };
  uint64_t thr = 0ull;          // keep keys >= thr
  bool keep_all = m >= n, keep_none = m <= 0;
  if (!keep_all && !keep_none) thr = block_select_kth_largest(n, m, key_of, hist, &s_prefix, &s_remaining);
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
      const int64_t j = q / T, t = q - j * T;
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
// row gather
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ x,
                                                          uint4 *__restrict__ x_perm,
                                                          const int32_t *__restrict__ row_token,
                                                          const int32_t *__restrict__ offsets, int E,
                                                          int64_t T, int vec_per_row,
                                                          uint32_t *err) {
  const int lane = threadIdx.x & 31;
  const int64_t R = offsets[E];
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += nwarps) {
    const int64_t t = row_token[r];
    if (t < 0 || t >= T) {
      if (lane == 0) raise_error(err, kErrBadIndex);
      continue;
    }
    const uint4 *src = x + t * vec_per_row;
    uint4 *dst = x_perm + r * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

cudaError_t launch_permute(const moe_config *c, const WsLayout &L, char *ws, const void *x,
                           const int32_t *topk_idx, const float *topk_gate, const float *probs,
                           int32_t *counts, int32_t *offsets, int32_t *tok_rows,
                           int32_t *row_token, float *row_gate, void *x_perm, int32_t *n_dropped,
                           cudaStream_t s) {
  uint32_t *err = reinterpret_cast<uint32_t *>(ws + L.err);
  const int E = c->E;
  const int64_t T = c->T;
  if (c->mode == MOE_EXPERT_CHOICE) {
    float *pt = reinterpret_cast<float *>(ws + L.probs_t);
    dim3 tb(32, 8), tg((unsigned)((T + 31) / 32), (unsigned)((E + 31) / 32));
    transpose_kernel<<<tg, tb, 0, s>>>(probs, pt, T, E);
    ec_select_kernel<<<E, 1024, 0, s>>>(pt, T, E, c->ec_capacity, counts, offsets, tok_rows,
                                        row_token, row_gate, n_dropped);
  } else {
    int32_t *hist = reinterpret_cast<int32_t *>(ws + L.hist);
    int32_t *base = reinterpret_cast<int32_t *>(ws + L.base);
    int32_t *cnt_off = reinterpret_cast<int32_t *>(ws + L.cnt_off);
    int32_t *kept = reinterpret_cast<int32_t *>(ws + L.kept);
    int32_t *sorted_q = reinterpret_cast<int32_t *>(ws + L.sorted_q);
    const int keepfrac = (c->capacity <= 0 && c->keep_den > 0) ? 1 : 0;
    hist_kernel<<<L.nblk, 256, 0, s>>>(topk_idx, T, c->k, E, hist, err);
    scan_kernel<<<1, 256, 0, s>>>(hist, L.nblk, E, T * c->k, c->capacity, c->keep_num, c->keep_den,
                                  base, counts, cnt_off, kept, offsets, n_dropped);
    rank_kernel<<<L.nblk, 256, 0, s>>>(topk_idx, topk_gate, T, c->k, E, base, offsets, cnt_off,
                                       c->capacity, keepfrac, tok_rows, row_token, row_gate,
                                       sorted_q);
    if (keepfrac)
      keep_select_kernel<<<E, 1024, 0, s>>>(sorted_q, cnt_off, kept, offsets, probs, topk_gate, T,
                                            c->k, E, tok_rows, row_token, row_gate);
  }
  const int vec_per_row = (int)(c->d_model * elem_size(c) / 16);
  const int64_t want = (L.rows_cap + 7) / 8;
  const int blocks = (int)std::min<int64_t>(want > 0 ? want : 1, (int64_t)sm_count() * 8);
  gather_rows_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4 *>(x),
                                            reinterpret_cast<uint4 *>(x_perm), row_token, offsets,
                                            E, T, vec_per_row, err);
  return cudaGetLastError();
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
// address is looked up once per device (with that device current) through
// cudaGetSymbolAddress and passed to the kernels like a workspace pointer.
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

// Device address of g_static_scratch on the current device.
cudaError_t static_scratch_address(char **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_address[dev] == nullptr) {
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
  if (L.step_end > kStaticScratchBytes) return MOE_ERR_WORKSPACE;   // beyond the fixed array
  const bool tc = cfg->mode == MOE_TOKEN_CHOICE;
  const bool keepfrac = tc && cfg->capacity <= 0 && cfg->keep_den > 0;
  if (!x || !counts || !offsets || !tok_rows || !row_token || !row_gate || !x_perm || !n_dropped)
    return MOE_ERR_INVALID_ARG;
  if (tc && (!topk_idx || !topk_gate)) return MOE_ERR_INVALID_ARG;
  if ((!tc || keepfrac) && !probs) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_perm) & 15u))
    return MOE_ERR_INVALID_ARG;
  char *scratch = nullptr;
  if (static_scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch + L.err, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e = launch_permute(cfg, L, scratch, x, topk_idx, topk_gate, probs, counts,
                                       offsets, tok_rows, row_token, row_gate, x_perm, n_dropped, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
