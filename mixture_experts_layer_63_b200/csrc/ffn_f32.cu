// fp32 expert FFN on CUDA cores, for layers whose dtype is fp32 (the
// tensor-core path is bf16).  Same grouped row layout as the tcgen05 path:
// routed expert e owns rows [offsets[e], offsets[e+1]) of x_perm / h /
// y_rows; shared expert s reads x and owns rows rows_cap + s*T + [0, T).
//   up   : h = ReLU(x W1^T)  or  SiLU(x W1^T) * (x W3^T)   (GShard section 3 /
//          SwiGLU of "大语言模型并行策略（七）：专家并行")
//   down : y_rows = G * (h W2^T), G = row gate (routed) or 1 (shared)
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int TM = 32, TN = 64, TK = 32;
constexpr int kMaxG = 320;

struct F32Params {
  int mode;                 // 0 relu, 1 swiglu, 2 scale (down-projection)
  int K, N;
  const float *a;           // routed A rows
  const float *a_static;    // static-group A rows
  int64_t a_static_base, a_static_stride;
  const float *b, *b3;      // [G * N, K]
  float *out;               // [*, N]
  const float *row_gate;
  const int32_t *offsets;
  int n_routed, n_static;
  int64_t rows_static, out_static_base;
  int64_t a_rows;
  uint32_t *err;
};

__global__ void __launch_bounds__(256) ffn_f32_kernel(const F32Params P) {
  __shared__ int s_prefix[kMaxG + 1];
  __shared__ int s_off[kMaxG], s_rows[kMaxG];
  __shared__ float As[TM][TK + 1];
  __shared__ float Bs[TN][TK + 1];
  __shared__ float B3s[TN][TK + 1];
  const int G = P.n_routed + P.n_static;
  const int nt = (P.N + TN - 1) / TN;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int g = 0; g < G; ++g) {
      int off = 0, rows;
      if (g < P.n_routed) {
        off = P.offsets[g];
        rows = P.offsets[g + 1] - off;
        if (rows < 0 || off < 0 || (int64_t)off + rows > P.a_rows) {
          raise_error(P.err, kErrBadIndex);
          rows = 0;
          off = 0;
        }
      } else {
        rows = (int)P.rows_static;
      }
      s_off[g] = off;
      s_rows[g] = rows;
      s_prefix[g] = acc;
      acc += ((rows + TM - 1) / TM) * nt;
    }
    s_prefix[G] = acc;
  }
  __syncthreads();
  const int total = s_prefix[G];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    int g = 0;
    while (g + 1 < G && s_prefix[g + 1] <= tile) ++g;
    const int local = tile - s_prefix[g];
    const int mt = (s_prefix[g + 1] - s_prefix[g]) / nt;
    const int n = local / mt, m = local - n * mt;
    const bool routed = g < P.n_routed;
    const float *A = routed ? P.a + ((int64_t)s_off[g] + (int64_t)m * TM) * P.K
                            : P.a_static + (P.a_static_base + (int64_t)(g - P.n_routed) * P.a_static_stride +
                                            (int64_t)m * TM) * P.K;
    const int rows_left = s_rows[g] - m * TM;
    const float *B = P.b + ((int64_t)g * P.N + (int64_t)n * TN) * P.K;
    const float *B3 = P.b3 ? P.b3 + ((int64_t)g * P.N + (int64_t)n * TN) * P.K : nullptr;
    const int cols_left = P.N - n * TN;
    float acc[2][4], acc3[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = acc3[i][j] = 0.f;
    for (int k0 = 0; k0 < P.K; k0 += TK) {
      __syncthreads();
      for (int i = threadIdx.x; i < TM * TK; i += 256) {
        const int r = i / TK, kk = i % TK;
        As[r][kk] = (r < rows_left && k0 + kk < P.K) ? A[(int64_t)r * P.K + k0 + kk] : 0.f;
      }
      for (int i = threadIdx.x; i < TN * TK; i += 256) {
        const int r = i / TK, kk = i % TK;
        const bool in = r < cols_left && k0 + kk < P.K;
        Bs[r][kk] = in ? B[(int64_t)r * P.K + k0 + kk] : 0.f;
        if (B3) B3s[r][kk] = in ? B3[(int64_t)r * P.K + k0 + kk] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < TK; ++kk) {
        const float a0 = As[ty * 2][kk], a1 = As[ty * 2 + 1][kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float bv = Bs[tx * 4 + j][kk];
          acc[0][j] = fmaf(a0, bv, acc[0][j]);
          acc[1][j] = fmaf(a1, bv, acc[1][j]);
          if (B3) {
            const float b3v = B3s[tx * 4 + j][kk];
            acc3[0][j] = fmaf(a0, b3v, acc3[0][j]);
            acc3[1][j] = fmaf(a1, b3v, acc3[1][j]);
          }
        }
      }
    }
    const int64_t out0 = routed ? (int64_t)s_off[g] + (int64_t)m * TM
                                : P.out_static_base + (int64_t)(g - P.n_routed) * P.rows_static + (int64_t)m * TM;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = ty * 2 + i;
      if (r >= rows_left) continue;
      float gate = 1.f;
      if (P.mode == 2 && routed) gate = P.row_gate[out0 + r];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = tx * 4 + j;
        if (c >= cols_left) continue;
        float v = acc[i][j];
        if (P.mode == 0) v = fmaxf(v, 0.f);
        else if (P.mode == 1) v = v / (1.f + expf(-v)) * acc3[i][j];
        else v = v * gate;
        P.out[(out0 + r) * P.N + (int64_t)n * TN + c] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_ffn_f32(const moe_config *c, const WsLayout &L, uint32_t *err, const float *x,
                           const float *x_perm,
                           const int32_t *offsets, const float *row_gate, const float *w1,
                           const float *w3, const float *w2, float *h, float *y_rows,
                           cudaStream_t s) {
  const int64_t T = c->T;
  const int grid = 148 * 4;
  F32Params up{};
  up.mode = c->act == MOE_ACT_SWIGLU ? 1 : 0;
  up.K = c->d_model;
  up.N = c->d_ff;
  up.a = x_perm;
  up.a_static = x;
  up.a_static_base = 0;
  up.a_static_stride = 0;
  up.b = w1;
  up.b3 = c->act == MOE_ACT_SWIGLU ? w3 : nullptr;
  up.out = h;
  up.offsets = offsets;
  up.n_routed = c->E;
  up.n_static = c->S;
  up.rows_static = T;
  up.out_static_base = L.rows_cap;
  up.a_rows = L.rows_cap;
  up.err = err;
  cudaError_t e = launch_kernel(ffn_f32_kernel, grid, 256, 0, s, up);
  if (e != cudaSuccess) return e;
  F32Params dn{};
  dn.mode = 2;
  dn.K = c->d_ff;
  dn.N = c->d_model;
  dn.a = h;
  dn.a_static = h;
  dn.a_static_base = L.rows_cap;
  dn.a_static_stride = T;
  dn.b = w2;
  dn.b3 = nullptr;
  dn.out = y_rows;
  dn.row_gate = row_gate;
  dn.offsets = offsets;
  dn.n_routed = c->E;
  dn.n_static = c->S;
  dn.rows_static = T;
  dn.out_static_base = L.rows_cap;
  dn.a_rows = L.rows_total;
  dn.err = err;
  return launch_kernel(ffn_f32_kernel, grid, 256, 0, s, dn);
}

}  // namespace moe
