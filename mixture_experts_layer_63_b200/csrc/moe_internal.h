// Internal host-side declarations of libmoe.so: kernel launchers and the
// workspace layout.  Not part of the public ABI (include/moe.h is).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Assignments per histogram block of the token-choice counting sort.
constexpr int kAssignBlock = 2048;
// Upper bound on routed experts and on top-k handled by the kernels.
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;

// Byte offsets into the caller's workspace.  The first region (error word +
// step scratch) is what the step entry points use; moe_forward adds its
// intermediates after it.
struct WsLayout {
  size_t err;        // uint32 error word (256 B reserved)
  size_t hist;       // int32 [nblk * E]   per-block expert histogram
  size_t base;       // int32 [nblk * E]   exclusive scan over blocks
  size_t cnt_off;    // int32 [E + 1]      exclusive scan of counts
  size_t kept;       // int32 [E]          rows kept per expert
  size_t sorted_q;   // int32 [T * k]      assignments grouped by expert (keep-fraction)
  size_t probs_t;    // fp32  [E * T]      transposed probabilities (expert choice)
  size_t step_end;
  // moe_forward intermediates
  size_t logits, probs, topk_idx, topk_gate, counts, offsets, n_dropped;
  size_t tok_rows, row_token, row_gate, x_perm, h, y_rows;
  size_t total;
  int nblk;          // histogram blocks
  int64_t rows_cap, rows_total, tok_rows_len;
};

moe_status validate(const moe_config *c);
WsLayout make_layout(const moe_config *c);

inline size_t elem_size(const moe_config *c) { return c->dtype == MOE_F32 ? 4 : 2; }

// --- router / gate (router_gate.cu) ---------------------------------------
cudaError_t launch_router_f32(const moe_config *c, const float *x, const float *w, const float *bias,
                              float *logits, cudaStream_t s);
cudaError_t launch_gate(const moe_config *c, const float *logits, float *probs, int32_t *topk_idx,
                        float *topk_gate, cudaStream_t s);

// --- permutation (permute.cu) ---------------------------------------------
cudaError_t launch_permute(const moe_config *c, const WsLayout &L, char *ws, const void *x,
                           const int32_t *topk_idx, const float *topk_gate, const float *probs,
                           int32_t *counts, int32_t *offsets, int32_t *tok_rows,
                           int32_t *row_token, float *row_gate, void *x_perm, int32_t *n_dropped,
                           cudaStream_t s);

// --- tcgen05 grouped GEMM (gemm_sm100.cu) ---------------------------------
enum GemmEpilogue : int {
  kEpiStoreF32 = 0,   // out fp32 = acc (+ bias[col])           (router logits)
  kEpiRelu = 1,       // out bf16 = relu(acc)                    (up-projection, ReLU)
  kEpiSwiglu = 2,     // out bf16 = silu(acc_gate) * acc_up      (gate/up projection)
  kEpiScale = 3,      // out fp32 = row_gate[row] * acc          (down-projection)
};

// One grouped GEMM  out[rows_g, N] = A[rows_g, K] . B_g[N, K]^T  per group g.
// Groups 0..n_routed-1 take their rows [offsets[g], offsets[g+1]) of A and of
// the output; groups n_routed..n_routed+n_static-1 ("static", e.g. shared
// experts) take rows_static rows starting at a_static_base + s*a_static_stride
// of A_static and out_static_base + s*rows_static of the output.
struct GroupedGemm {
  int epi;
  int K;                    // contraction size (multiple of 64)
  int N;                    // output columns per group (weight rows per group)
  const void *a;            // bf16 [a_rows, K]
  int64_t a_rows;
  const void *a_static;     // bf16 [a_static_rows, K]
  int64_t a_static_rows;
  const void *b;            // bf16 [n_groups_w * N, K]  (w1 / w2 / router)
  const void *b3;           // bf16, SwiGLU up-projection weights, same shape as b
  int64_t b_rows;
  const int32_t *offsets;   // device [n_routed + 1] (may be null when n_routed == 0)
  int n_routed;
  int n_static;
  int64_t rows_static;
  int64_t a_static_base, a_static_stride;
  int64_t out_static_base;
  int64_t max_routed_rows;  // host upper bound of offsets[n_routed] (grid sizing)
  void *out;                // [*, N] row-major, ld = N
  const float *row_gate;    // kEpiScale: gate per routed output row
  const float *bias;        // kEpiStoreF32: [N] or null
  uint32_t *err;
};
cudaError_t launch_grouped_gemm(const GroupedGemm &g, cudaStream_t s);

// --- fp32 CUDA-core expert FFN (ffn_f32.cu) ----------------------------------
cudaError_t launch_ffn_f32(const moe_config *c, const WsLayout &L, uint32_t *err, const float *x,
                           const float *x_perm,
                           const int32_t *offsets, const float *row_gate, const float *w1,
                           const float *w3, const float *w2, float *h, float *y_rows,
                           cudaStream_t s);

// --- combine (combine.cu) ----------------------------------------------------
cudaError_t launch_combine(const moe_config *c, int64_t rows_cap, const void *y_rows,
                           const int32_t *tok_rows, void *y, cudaStream_t s);

}  // namespace moe
