// Gate-weighted combine (GShard section 3 of "MoE技术演进": y_s = sum_e
// G_{s,e} FFN_e(x_s); DeepSeekMoE section 2: plus the shared experts' sum).
// The gates were applied in the down-projection epilogue, which leaves rows
// in the layer dtype; here each token sums its rows: routed rows in the
// token's k-rank order (expert choice: ascending expert), then shared experts
// 0..S-1, fp32 accumulation, one rounding to the output dtype.  One warp per
// token, 16-byte vectors.  (moe_forward with at most two rows a token adds
// the rows into y in the down-projection's epilogue instead, with the same
// result; this kernel then does not run.)
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxRows = kMaxExperts + 16;
#ifndef MOE_COMBINE_BATCH
#define MOE_COMBINE_BATCH 8
#endif
constexpr int kRowBatch = MOE_COMBINE_BATCH;    // rows loaded before they are added

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32) combine_kernel(const void *__restrict__ y_rows,
                                                              const int32_t *__restrict__ tok_rows,
                                                              void *__restrict__ y, int64_t T, int d,
                                                              int W, int expert_major, int S,
                                                              int64_t rows_cap) {
  __shared__ int s_rows[kWarps][kMaxRows];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
  pdl_wait();
  pdl_trigger();
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

  // one 16-byte vector per lane and step: 8 bf16 or 4 fp32 elements; the
  // token's rows are loaded eight at a time before they are added (in row
  // order), so a lane keeps up to eight loads in flight
  constexpr int EPV = BF16 ? 8 : 4;
  const int nvec = d / EPV;
  const uint4 *src = reinterpret_cast<const uint4 *>(y_rows);
  for (int v = lane; v < nvec; v += 32) {
    float acc[EPV];
#pragma unroll
    for (int i = 0; i < EPV; ++i) acc[i] = 0.f;
    for (int i0 = 0; i0 < n; i0 += kRowBatch) {
      uint4 a[kRowBatch];
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i)
        if (i0 + i < n) a[i] = src[(int64_t)rows[i0 + i] * nvec + v];
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i) {
        if (i0 + i < n) {
          if (BF16) {
            acc[0] += bf16_lo(a[i].x); acc[1] += bf16_hi(a[i].x);
            acc[2 % EPV] += bf16_lo(a[i].y); acc[3 % EPV] += bf16_hi(a[i].y);
            acc[4 % EPV] += bf16_lo(a[i].z); acc[5 % EPV] += bf16_hi(a[i].z);
            acc[6 % EPV] += bf16_lo(a[i].w); acc[7 % EPV] += bf16_hi(a[i].w);
          } else {
            acc[0] += __uint_as_float(a[i].x);
            acc[1] += __uint_as_float(a[i].y);
            acc[2 % EPV] += __uint_as_float(a[i].z);
            acc[3 % EPV] += __uint_as_float(a[i].w);
          }
        }
      }
    }
    if (BF16) {
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4 % EPV], acc[5 % EPV]);
      o.w = pack_bf16x2(acc[6 % EPV], acc[7 % EPV]);
      reinterpret_cast<uint4 *>(y)[t * nvec + v] = o;
    } else {
      reinterpret_cast<float4 *>(y)[t * nvec + v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config *c, int64_t rows_cap, const void *y_rows,
                           const int32_t *tok_rows, void *y, cudaStream_t s) {
  const bool ec = c->mode == MOE_EXPERT_CHOICE;
  const int W = ec ? c->E : c->k;
  const unsigned blocks = (unsigned)((c->T + kWarps - 1) / kWarps);
  auto kern = c->dtype == MOE_BF16 ? combine_kernel<true> : combine_kernel<false>;
  return launch_kernel(kern, blocks, kWarps * 32, 0, s, y_rows, tok_rows, y, c->T, c->d_model, W,
                       ec ? 1 : 0, c->S, rows_cap);
}

}  // namespace moe
