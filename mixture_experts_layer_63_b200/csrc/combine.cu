// Gate-weighted combine (GShard section 3 of "MoE技术演进": y_s = sum_e
// G_{s,e} FFN_e(x_s); DeepSeekMoE section 2: plus the shared experts' sum).
// The gates were applied in the down-projection epilogue, so here each
// token sums its rows: routed rows in the token's k-rank order (expert
// choice: ascending expert), then shared experts 0..S-1, fp32 accumulation,
// one rounding to the output dtype.  One warp per token, 16-byte vectors.
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxRows = kMaxExperts + 16;

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) combine_kernel(const void *__restrict__ y_rows,
                                                              const int32_t *__restrict__ tok_rows,
                                                              void *__restrict__ y, int64_t T, int d,
                                                              int W, int expert_major, int S,
                                                              int64_t rows_cap) {
  __shared__ int s_rows[kWarps][kMaxRows];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
  if (t >= T) return;
  int *rows = s_rows[warp];
  // collect the token's rows in order
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

  const int epv = BF16 ? 8 : 4;                 // elements per 16-byte vector
  const int nvec = d / epv;
  const uint4 *src = reinterpret_cast<const uint4 *>(y_rows);
  uint4 *dst = reinterpret_cast<uint4 *>(y);
  for (int v = lane; v < nvec; v += 32) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int i = 0; i < n; ++i) {
      const uint4 q = src[(int64_t)rows[i] * nvec + v];
      if (BF16) {
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      } else {
        acc[0] += __uint_as_float(q.x); acc[1] += __uint_as_float(q.y);
        acc[2] += __uint_as_float(q.z); acc[3] += __uint_as_float(q.w);
      }
    }
    uint4 o;
    if (BF16) {
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
    } else {
      o.x = __float_as_uint(acc[0]);
      o.y = __float_as_uint(acc[1]);
      o.z = __float_as_uint(acc[2]);
      o.w = __float_as_uint(acc[3]);
    }
    dst[t * nvec + v] = o;
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config *c, int64_t rows_cap, const void *y_rows,
                           const int32_t *tok_rows, void *y, cudaStream_t s) {
  const bool ec = c->mode == MOE_EXPERT_CHOICE;
  const int W = ec ? c->E : c->k;
  const unsigned blocks = (unsigned)((c->T + kWarps - 1) / kWarps);
  if (c->dtype == MOE_BF16)
    combine_kernel<true><<<blocks, kWarps * 32, 0, s>>>(y_rows, tok_rows, y, c->T, c->d_model, W,
                                                        ec ? 1 : 0, c->S, rows_cap);
  else
    combine_kernel<false><<<blocks, kWarps * 32, 0, s>>>(y_rows, tok_rows, y, c->T, c->d_model, W,
                                                         ec ? 1 : 0, c->S, rows_cap);
  return cudaGetLastError();
}

}  // namespace moe
