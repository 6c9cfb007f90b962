// Backward pass of the layer (training), bf16 layers: gradients of
// L = sum(dy * y) for x, the router weights (and logit bias) and every
// expert's W1 / W3 / W2, with the routing decisions of the forward held fixed.
//
// The pages train these layers (GShard, DeepSeekMoE, DeepSeek-V2/V3 in
// "MoE技术演进"; the softmax gating network of "Adaptive Mixtures of Local
// Experts"): experts receive gradient through their kept rows, the router
// through the gate G of each kept row (G = p, p / sum of the selected p when
// renormalised, s + b under DeepSeek-V3's bias routing).
//
// This file holds the data-movement and small arithmetic kernels; the
// contractions run on the tcgen05 grouped GEMM (gemm_sm100.cu):
//   recompute    A|U = X . [W1|W3]^T            (pre-activations, bf16)
//   dact         dA|dU = act'(A, U) * (g * dY . W2)      (fused epilogue;
//                W2 read as it is stored, MN-major)
//   dX rows      dX = [dA|dU] . [W1;W3]          (fp32 rows, summed per token;
//                W1, W3 read MN-major)
//   wgrad        dW2_e = (g dY)_e^T H_e,  [dW1|dW3]_e = [dA|dU]_e^T X_e
//                (K-grouped: each expert contracts over its own rows)
//   router       dW_r = dl^T X,  dx += dl . W_r   (dl from the gate gradients)
// The weight-gradient operands are transposed here into 64-padded segments
// (an expert's rows are not 64-aligned in the forward's row layout).
#include <algorithm>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// ---- tiled transposes (64 x 64 bf16 tiles through shared memory) ----------
// A tile is read as 16-byte vectors along its rows (8 elements) and written
// as 16-byte vectors along its columns; partial vectors at a ragged edge
// fall back to single elements.
constexpr int kTT = 64;                 // tile edge
constexpr int kTP = kTT + 2;            // shared-memory row pitch (halfs): spreads the banks

struct TileIO {
  // source row r of the tile (-1: zeros) and its factor
  int64_t row;
  float scale;
};

__device__ __forceinline__ void tile_load_row(uint16_t (*tile)[kTP], int i, const uint16_t *src_row,
                                              int c0, int C, int v, float scale) {
  // 8 elements c0 + 8v .. c0 + 8v + 7 of one source row into tile[i][8v..]
  const int c = c0 + 8 * v;
  uint16_t e[8];
  if (src_row && c + 8 <= C && ((reinterpret_cast<uintptr_t>(src_row + c) & 15) == 0)) {
    const uint4 q = *reinterpret_cast<const uint4 *>(src_row + c);
    e[0] = (uint16_t)(q.x & 0xffff); e[1] = (uint16_t)(q.x >> 16);
    e[2] = (uint16_t)(q.y & 0xffff); e[3] = (uint16_t)(q.y >> 16);
    e[4] = (uint16_t)(q.z & 0xffff); e[5] = (uint16_t)(q.z >> 16);
    e[6] = (uint16_t)(q.w & 0xffff); e[7] = (uint16_t)(q.w >> 16);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) e[j] = (src_row && c + j < C) ? src_row[c + j] : (uint16_t)0;
  }
  if (scale != 1.0f) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      e[j] = __bfloat16_as_ushort(__float2bfloat16_rn(scale * __bfloat162float(__ushort_as_bfloat16(e[j]))));
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) tile[i][8 * v + j] = e[j];
}

// out row (tile column) c: 8 consecutive tile rows 8v .. 8v+7 at dst[8v..]
__device__ __forceinline__ void tile_store_col(uint16_t (*tile)[kTP], int c, uint16_t *dst, int v,
                                               int nrows) {
  uint16_t e[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) e[j] = tile[8 * v + j][c];
  if (8 * v + 8 <= nrows && ((reinterpret_cast<uintptr_t>(dst + 8 * v) & 15) == 0)) {
    uint4 q;
    q.x = (uint32_t)e[0] | ((uint32_t)e[1] << 16);
    q.y = (uint32_t)e[2] | ((uint32_t)e[3] << 16);
    q.z = (uint32_t)e[4] | ((uint32_t)e[5] << 16);
    q.w = (uint32_t)e[6] | ((uint32_t)e[7] << 16);
    *reinterpret_cast<uint4 *>(dst + 8 * v) = q;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (8 * v + j < nrows) dst[8 * v + j] = e[j];
  }
}

// out[b][c][col_off + r] = in[b][r][c] for r < R, c < C (bf16), 256 threads
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t *__restrict__ in,
                                                             uint16_t *__restrict__ out, int R, int C,
                                                             int64_t ld_in, int64_t ld_out,
                                                             int64_t bstride_in, int64_t bstride_out,
                                                             int col_off) {
  __shared__ uint16_t tile[kTT][kTP];
  pdl_wait();
  pdl_trigger();
  const int64_t b = blockIdx.z;
  const int r0 = blockIdx.x * kTT, c0 = blockIdx.y * kTT;
  const uint16_t *src = in + b * bstride_in;
  uint16_t *dst = out + b * bstride_out;
  for (int k = threadIdx.x; k < kTT * 8; k += blockDim.x) {
    const int i = k >> 3, v = k & 7;
    const int r = r0 + i;
    tile_load_row(tile, i, r < R ? src + (int64_t)r * ld_in : nullptr, c0, C, v, 1.0f);
  }
  __syncthreads();
  const int nrows = min(kTT, R - r0);
  for (int k = threadIdx.x; k < kTT * 8; k += blockDim.x) {
    const int c = k >> 3, v = k & 7;
    if (c0 + c < C) tile_store_col(tile, c, dst + (int64_t)(c0 + c) * ld_out + col_off + r0, v, nrows);
  }
}

// fp32 [R, C] -> bf16 [C][ld_out] (zero padding to ld_out), for dl^T
__global__ void transpose_f32_to_bf16_kernel(const float *__restrict__ in, __nv_bfloat16 *__restrict__ out,
                                             int R, int C, int Rpad, int64_t ld_out) {
  __shared__ float tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int r0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < R && c < C) ? in[(int64_t)r * C + c] : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < C && r < Rpad) out[(int64_t)c * ld_out + r] = __float2bfloat16_rn(tile[threadIdx.x][i]);
  }
}

// ---- segments of the K-grouped weight gradients --------------------------
// kseg[g] = sum over g' < g of round_up(len_g', 64): routed expert e has
// offsets[e+1] - offsets[e] rows, each shared expert T rows.
__global__ void seg_offsets_kernel(const int32_t *__restrict__ offsets, int E, int S, int64_t T,
                                   int32_t *__restrict__ kseg) {
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int acc = 0;
  for (int g = 0; g < E + S; ++g) {
    kseg[g] = acc;
    const int len = g < E ? offsets[g + 1] - offsets[g] : (int)T;
    acc += (len + 63) / 64 * 64;
  }
  kseg[E + S] = acc;
}

// out[c][kseg[g] + i] = scale_i * src[row_i][c] for the rows i of group g
// (zeros in the padding up to the next segment).  Row i of routed group e
// is r = offsets[e] + i, read at map[r] (null: r); scale_i = scale[r] (null:
// 1).  Row i of shared group s is read at shared_base + s * shared_stride + i.
// 64 x 64 tiles: segments are 64-aligned, so a tile never straddles two.
constexpr int kMaxSegGroups = kMaxExperts + 8;         // routed + shared experts
struct SegSrc {
  const __nv_bfloat16 *src;
  int64_t ld;                // elements per source row
  const int32_t *map;        // routed rows: source row of row r (or null)
  const float *scale;        // routed rows: factor (or null)
  int64_t shared_base, shared_stride;
};

__global__ void __launch_bounds__(256) transpose_segments_kernel(SegSrc S_, const int32_t *__restrict__ offsets,
                                                                 const int32_t *__restrict__ kseg,
                                                                 int E, int G, int C, int64_t ld_out,
                                                                 __nv_bfloat16 *__restrict__ out,
                                                                 uint32_t *err, int64_t src_rows,
                                                                 int64_t shared_len) {
  __shared__ uint16_t tile[kTT][kTP];
  __shared__ int64_t s_row[kTT];
  __shared__ float s_scale[kTT];
  __shared__ int s_kseg[kMaxSegGroups + 1];
  pdl_wait();
  pdl_trigger();
  const int k0 = blockIdx.x * kTT, c0 = blockIdx.y * kTT;
  // the segment offsets into shared memory in one parallel load, so that the
  // search below costs no chain of dependent global loads
  for (int i = threadIdx.x; i <= G; i += blockDim.x) s_kseg[i] = kseg[i];
  __syncthreads();
  if (k0 >= s_kseg[G]) return;                          // past the last segment
  int lo = 0, hi = G - 1;                               // group holding column k0
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_kseg[mid] <= k0) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int64_t len = g < E ? (int64_t)(offsets[g + 1] - offsets[g]) : shared_len;
  if (threadIdx.x < kTT) {
    const int64_t li = (int64_t)(k0 - s_kseg[g]) + threadIdx.x;  // row of the segment
    int64_t row = -1;
    float sc = 1.0f;
    if (li < len) {
      if (g < E) {
        const int64_t r = (int64_t)offsets[g] + li;
        row = S_.map ? S_.map[r] : r;
        if (S_.scale) sc = S_.scale[r];
      } else {
        row = S_.shared_base + (int64_t)(g - E) * S_.shared_stride + li;
      }
      if (row < 0 || row >= src_rows) {
        raise_error(err, kErrBadIndex);
        row = -1;
      }
    }
    s_row[threadIdx.x] = row;
    s_scale[threadIdx.x] = sc;
  }
  __syncthreads();
  const uint16_t *src = reinterpret_cast<const uint16_t *>(S_.src);
  for (int k = threadIdx.x; k < kTT * 8; k += blockDim.x) {
    const int i = k >> 3, v = k & 7;
    const int64_t row = s_row[i];
    tile_load_row(tile, i, row >= 0 ? src + row * S_.ld : nullptr, c0, C, v, s_scale[i]);
  }
  __syncthreads();
  uint16_t *dst = reinterpret_cast<uint16_t *>(out);
  for (int k = threadIdx.x; k < kTT * 8; k += blockDim.x) {
    const int c = k >> 3, v = k & 7;
    if (c0 + c < C) tile_store_col(tile, c, dst + (int64_t)(c0 + c) * ld_out + k0, v, kTT);
  }
}

// ---- gathers --------------------------------------------------------------
// dst[r] = src[map[r]] for r < offsets[E] (bf16 rows of d elements), one warp per row
__global__ void __launch_bounds__(256) gather_bf16_rows_kernel(const uint4 *__restrict__ src,
                                                               uint4 *__restrict__ dst,
                                                               const int32_t *__restrict__ map,
                                                               const int32_t *__restrict__ offsets,
                                                               int E, int64_t src_rows, int vpr,
                                                               uint32_t *err) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t R = offsets[E];
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += nw) {
    const int64_t t = map[r];
    if (t < 0 || t >= src_rows) {
      if (lane == 0) raise_error(err, kErrBadIndex);
      continue;
    }
    for (int v = lane; v < vpr; v += 32) dst[r * vpr + v] = src[t * vpr + v];
  }
}

// ---- gate gradients and the router ---------------------------------------
// dG_r = <dy[t], FFN_e(x_t)> for each kept routed row r of token t.  With
// FFN_e(x) = W2_e h, this is <dy[t] W2_e, h_r>: the dact GEMM, whose
// accumulator holds dy[t] W2_e, multiplies it by h in its epilogue (ReLU:
// relu of the recomputed a, which equals the forward's rounded h; SwiGLU:
// the forward's h itself) and leaves one partial sum per 256-column N-tile;
// here they are added in N-tile order.
__global__ void __launch_bounds__(256) gate_grad_kernel(const float *__restrict__ dg_part, int nt,
                                                        const int32_t *__restrict__ offsets, int E,
                                                        float *__restrict__ dgate) {
  pdl_wait();
  pdl_trigger();
  const int64_t R = offsets[E];
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R;
       r += (int64_t)gridDim.x * blockDim.x) {
    const float *p = dg_part + r * nt;
    float acc = p[0];
    for (int n = 1; n < nt; ++n) acc = __fadd_rn(acc, p[n]);
    dgate[r] = acc;
  }
}

// Per token (one warp): dp from the gate gradients of its kept rows, then
// dl = p * (dp - <p, dp>).  Token choice: the k selected experts' gate
// sources s_j (p, or p + b under bias routing); renormalised gates
// G_j = s_j / S give dL/ds_i = (dG_i - sum_j dG_j G_j) / S.  Expert choice:
// dp[t, e] = dG of the row (e, t).
__global__ void __launch_bounds__(256) router_grad_kernel(const float *__restrict__ probs,
                                                          const int32_t *__restrict__ topk_idx,
                                                          const int32_t *__restrict__ tok_rows,
                                                          const float *__restrict__ dgate,
                                                          const float *__restrict__ state, int64_t T,
                                                          int E, int k, int expert_choice, int rule,
                                                          int renormalize, float *__restrict__ dl) {
  __shared__ float s_dp[8][kMaxExperts];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * 8 + w;
  if (t >= T) return;
  float *dp = s_dp[w];
  for (int e = lane; e < E; e += 32) dp[e] = 0.0f;
  __syncwarp();
  const float *p = probs + t * E;
  if (expert_choice) {
    for (int e = lane; e < E; e += 32) {
      const int r = tok_rows[(int64_t)e * T + t];
      dp[e] = r >= 0 ? dgate[r] : 0.0f;
    }
  } else if (lane == 0) {
    float src[kMaxTopK], dg[kMaxTopK];
    int ix[kMaxTopK];
    float S = 0.0f;
    for (int j = 0; j < k; ++j) {
      ix[j] = topk_idx[t * k + j];
      src[j] = p[ix[j]] + (rule == 1 ? state[ix[j]] : 0.0f);
      S += src[j];
      const int r = tok_rows[t * k + j];
      dg[j] = r >= 0 ? dgate[r] : 0.0f;
    }
    if (renormalize) {
      float dot = 0.0f;
      for (int j = 0; j < k; ++j) dot += dg[j] * (src[j] / S);
      for (int j = 0; j < k; ++j) dp[ix[j]] += (dg[j] - dot) / S;
    } else {
      for (int j = 0; j < k; ++j) dp[ix[j]] += dg[j];
    }
  }
  __syncwarp();
  float dot = 0.0f;
  for (int e = lane; e < E; e += 32) dot += p[e] * dp[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  for (int e = lane; e < E; e += 32) dl[t * E + e] = p[e] * (dp[e] - dot);
}

// dbias[e] = sum_t dl[t, e], one block per expert, fixed summation order
__global__ void __launch_bounds__(256) bias_grad_kernel(const float *__restrict__ dl, int64_t T, int E,
                                                        float *__restrict__ dbias) {
  __shared__ float s[256];
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x;
  float acc = 0.0f;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) acc += dl[t * E + e];
  s[threadIdx.x] = acc;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) s[threadIdx.x] += s[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) dbias[e] = s[0];
}

// dx[t] = sum of t's routed dX rows (k-rank order; expert choice: ascending
// expert) + its shared rows + the router term dx_router[t], fp32; one warp
// per token
__global__ void __launch_bounds__(256) dx_finish_kernel(const float *__restrict__ dx_rows,
                                                        const int32_t *__restrict__ tok_rows,
                                                        const float *__restrict__ dx_router,
                                                        float *__restrict__ dx, int64_t T, int d,
                                                        int W, int expert_major, int S,
                                                        int64_t rows_cap) {
  __shared__ int s_rows[8][kMaxExperts + 16];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * 8 + warp;
  if (t >= T) return;
  int *rows = s_rows[warp];
  int n = 0;
  for (int c = 0; c < W; c += 32) {
    const int w = c + lane;
    int r = -1;
    if (w < W) r = expert_major ? tok_rows[(int64_t)w * T + t] : tok_rows[t * W + w];
    const unsigned valid = __ballot_sync(0xffffffffu, r >= 0);
    if (r >= 0) rows[n + __popc(valid & ((1u << lane) - 1u))] = r;
    n += __popc(valid);
  }
  if (lane < S) rows[n + lane] = (int)(rows_cap + (int64_t)lane * T + t);
  n += S;
  __syncwarp();
  const int nv = d / 4;
  const float4 *src = reinterpret_cast<const float4 *>(dx_rows);
  const float4 *rt = reinterpret_cast<const float4 *>(dx_router) + t * nv;
  float4 *out = reinterpret_cast<float4 *>(dx) + t * nv;
  for (int v = lane; v < nv; v += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < n; ++i) {
      const float4 a = src[(int64_t)rows[i] * nv + v];
      acc.x += a.x; acc.y += a.y; acc.z += a.z; acc.w += a.w;
    }
    const float4 b = rt[v];
    acc.x += b.x; acc.y += b.y; acc.z += b.z; acc.w += b.w;
    out[v] = acc;
  }
}

}  // namespace

// ---- launchers ----------------------------------------------------------
cudaError_t launch_transpose_bf16(const void *in, void *out, int R, int C, int64_t ld_in,
                                  int64_t ld_out, int batch, int64_t bstride_in,
                                  int64_t bstride_out, int col_off, cudaStream_t s) {
  dim3 grid((unsigned)((R + kTT - 1) / kTT), (unsigned)((C + kTT - 1) / kTT), (unsigned)batch),
      block(256);
  return launch_kernel(transpose_bf16_kernel, grid, block, 0, s, static_cast<const uint16_t *>(in),
                       static_cast<uint16_t *>(out), R, C, ld_in, ld_out, bstride_in, bstride_out,
                       col_off);
}

cudaError_t launch_transpose_f32_bf16(const float *in, void *out, int R, int C, int Rpad,
                                      int64_t ld_out, cudaStream_t s) {
  dim3 grid((unsigned)((Rpad + 31) / 32), (unsigned)((C + 31) / 32)), block(32, 8);
  return launch_kernel(transpose_f32_to_bf16_kernel, grid, block, 0, s, in,
                       static_cast<__nv_bfloat16 *>(out), R, C, Rpad, ld_out);
}

cudaError_t launch_seg_offsets(const int32_t *offsets, int E, int S, int64_t T, int32_t *kseg,
                               cudaStream_t s) {
  return launch_kernel(seg_offsets_kernel, 1, 32, 0, s, offsets, E, S, T, kseg);
}

cudaError_t launch_transpose_segments(const void *src, int64_t ld, const int32_t *map,
                                      const float *scale, int64_t shared_base, int64_t shared_stride,
                                      int64_t shared_len, int64_t src_rows, const int32_t *offsets,
                                      const int32_t *kseg,
                                      int E, int G, int C, int64_t kp_max, void *out, uint32_t *err,
                                      cudaStream_t s) {
  if (G < 1 || G > kMaxSegGroups) return cudaErrorInvalidValue;
  SegSrc S_{static_cast<const __nv_bfloat16 *>(src), ld, map, scale, shared_base, shared_stride};
  dim3 grid((unsigned)(kp_max / kTT), (unsigned)((C + kTT - 1) / kTT)), block(256);
  return launch_kernel(transpose_segments_kernel, grid, block, 0, s, S_, offsets, kseg, E, G, C,
                       kp_max, static_cast<__nv_bfloat16 *>(out), err, src_rows, shared_len);
}

cudaError_t launch_gather_bf16_rows(const void *src, void *dst, const int32_t *map,
                                    const int32_t *offsets, int E, int64_t src_rows, int d,
                                    int64_t max_rows, uint32_t *err, cudaStream_t s) {
  const int64_t want = (max_rows + 7) / 8;
  const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, 148 * 8));
  return launch_kernel(gather_bf16_rows_kernel, blocks, 256, 0, s, static_cast<const uint4 *>(src),
                       static_cast<uint4 *>(dst), map, offsets, E, src_rows, d / 8, err);
}

cudaError_t launch_gate_grad(const float *dg_part, int nt, const int32_t *offsets, int E,
                             int64_t max_rows, float *dgate, cudaStream_t s) {
  const int64_t want = (max_rows + 255) / 256;
  const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, 148 * 8));
  return launch_kernel(gate_grad_kernel, blocks, 256, 0, s, dg_part, nt, offsets, E, dgate);
}

cudaError_t launch_router_grad(const moe_config *c, const float *probs, const int32_t *topk_idx,
                               const int32_t *tok_rows, const float *dgate, const float *state,
                               float *dl, cudaStream_t s) {
  const bool ec = c->mode == MOE_EXPERT_CHOICE;
  const unsigned blocks = (unsigned)((c->T + 7) / 8);
  return launch_kernel(router_grad_kernel, blocks, 256, 0, s, probs, topk_idx, tok_rows, dgate,
                       state, c->T, c->E, ec ? 0 : c->k, ec ? 1 : 0,
                       ec ? 0 : c->route_rule, ec ? 0 : c->renormalize, dl);
}

cudaError_t launch_bias_grad(const float *dl, int64_t T, int E, float *dbias, cudaStream_t s) {
  return launch_kernel(bias_grad_kernel, (unsigned)E, 256, 0, s, dl, T, E, dbias);
}

cudaError_t launch_dx_finish(const moe_config *c, int64_t rows_cap, const float *dx_rows,
                             const int32_t *tok_rows, const float *dx_router, float *dx,
                             cudaStream_t s) {
  const bool ec = c->mode == MOE_EXPERT_CHOICE;
  const unsigned blocks = (unsigned)((c->T + 7) / 8);
  return launch_kernel(dx_finish_kernel, blocks, 256, 0, s, dx_rows, tok_rows, dx_router, dx, c->T,
                       c->d_model, ec ? c->E : c->k, ec ? 1 : 0, c->S, rows_cap);
}

}  // namespace moe

namespace moe {
namespace {
// out[r][c] = bf16(in[r][c]) for c < C, 0 for C <= c < Cp
__global__ void pad_f32_to_bf16_kernel(const float *__restrict__ in, __nv_bfloat16 *__restrict__ out,
                                       int64_t R, int C, int Cp) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = R * Cp;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / Cp;
    const int c = (int)(i - r * Cp);
    out[i] = __float2bfloat16_rn(c < C ? in[r * C + c] : 0.0f);
  }
}
}  // namespace

cudaError_t launch_pad_f32_bf16(const float *in, void *out, int64_t R, int C, int Cp,
                                cudaStream_t s) {
  const int64_t n = R * Cp;
  const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 8));
  return launch_kernel(pad_f32_to_bf16_kernel, blocks, 256, 0, s, in,
                       static_cast<__nv_bfloat16 *>(out), R, C, Cp);
}

}  // namespace moe
