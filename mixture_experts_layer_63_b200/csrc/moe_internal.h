// Internal host-side declarations of libmoe.so: kernel launchers and the
// workspace layout.  Not part of the public ABI (include/moe.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Launch `kern` on `s` with programmatic stream serialization, so that its
// CTAs may start while the previous kernel on the stream finishes (the
// kernels call pdl_wait() before touching global memory).  MOE_PDL=0 at
// build time launches with plain stream order instead.
#ifndef MOE_PDL
#define MOE_PDL 1
#endif
// Kernels this library has launched, all threads together (moe_kernel_launches).
void count_launch();

template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = MOE_PDL ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e == cudaSuccess) count_launch();
  return e;
}

// Tokens per unit of the token-choice counting sort (one warp per unit).
constexpr int kUnitTokens = 32;
constexpr int kUnitsPerBlock = 32;      // units per block of the permutation's scans

// Numbering of the token-choice units.  Tokens form G local groups (GShard's
// local group dispatch; G = 1 without it) of nbg 32-token blocks each; unit
// u = g*upg + r*nbg + bl holds the rank-r choices of block bl of group g
// (upg = k*nbg units per group), so a group's units are contiguous and in its
// own priority order.  Scan blocks of kUnitsPerBlock units never straddle a
// group: bpg blocks per group, nb in all.
struct UnitGrid {
  int G, nbg, upg, bpg, nb;
};
inline UnitGrid unit_grid(const moe_config *c) {
  UnitGrid u;
  u.G = c->local_groups > 1 ? c->local_groups : 1;
  u.nbg = u.G > 1 ? (int)(c->T / u.G / kUnitTokens) : (int)((c->T + kUnitTokens - 1) / kUnitTokens);
  u.upg = (c->mode == MOE_TOKEN_CHOICE ? c->k : 0) * u.nbg;
  u.bpg = (u.upg + kUnitsPerBlock - 1) / kUnitsPerBlock;
  u.nb = u.G * u.bpg;
  return u;
}
// Upper bound on routed experts and on top-k handled by the kernels.
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
// The router runs inside the gate kernel when E <= 32 and W_r, widened to
// fp32, fits this many bytes of shared memory; otherwise the tcgen05 GEMM
// (bf16) or a CUDA-core kernel (fp32) computes the logits first.
constexpr size_t kFusedRouterSmem = 200 * 1024;

// Byte offsets into the caller's workspace.  The first region (error word +
// step scratch) is what the step entry points use; moe_forward adds its
// intermediates after it.
// Control block at the start of every workspace: the uint32 error word at
// offset 0 and the stream-K ready flags (int32 [kSkSlots]) at kSkFlagsOffset.
// All zero in a fresh workspace; kernels leave the flags at zero when they
// finish without an error.
constexpr size_t kCtrlBytes = 4096;
constexpr size_t kSkFlagsOffset = 256;
constexpr int kSkSlots = 192;                 // stream-K slots: >= CTAs of one GEMM launch
constexpr int kSkSlotFloats = 128 * 256;      // one CTA's fp32 accumulator tile

struct WsLayout {
  size_t err;        // control block (kCtrlBytes): error word, stream-K flags
  size_t hist;       // int32 [k * nunit * E]  per-unit expert histogram
  size_t base;       // int32 [ceil(k * nunit / 32) * E]  per-expert totals of 32-unit blocks
  size_t cnt_off;    // int32 [E + 1]      exclusive scan of counts
  size_t kept;       // int32 [E]          rows kept per expert
  size_t sorted_q;   // int32 [T * k]      assignments grouped by expert (keep-fraction)
  size_t probs_t;    // fp32  [E * T]      transposed probabilities (expert choice)
  size_t permute_end;    // end of the permutation's scratch
  size_t logits_part;    // fp32 [ksplit][T][E] partial router logits (bf16 router with split K)
  size_t sk_part;        // fp32 [kSkSlots][kSkSlotFloats] stream-K partial tiles (bf16 GEMMs)
  size_t step_end;
  // moe_forward intermediates
  size_t logits, probs, topk_idx, topk_gate, counts, offsets, n_dropped;
  size_t tok_rows, row_token, row_gate, x_perm, h, y_rows;
  size_t total;
  // moe_forward_host staging rows of x and y (after everything moe_forward uses)
  size_t x_stage, y_stage, host_total;
  int nunit;         // 32-token units: ceil(T / 32)
  int64_t rows_cap, rows_total, tok_rows_len;
};

moe_status validate(const moe_config *c);
WsLayout make_layout(const moe_config *c);
// expert capacity C per (local group and) routed expert from the capacity
// factor, exact ceiling, clamped to the group's tokens; 0 = unlimited
int64_t capacity_rows(const moe_config *c);

inline size_t elem_size(const moe_config *c) { return c->dtype == MOE_F32 ? 4 : 2; }

// --- router / gate (router_gate.cu) ---------------------------------------
// true when the gate kernel computes the logits itself (small E)
bool router_is_fused(const moe_config *c);
// Gate (+ histogram for token choice).  logits_in == null: fused router from
// x and w_router, writing logits_out; else gate on the given logits.
// logits_in may hold nsplit partial sums split_stride floats apart (summed in
// order, then + bias when bias is given).
// state: the per-expert routing bias or utilisation of c->route_rule (or null).
// y_zero non-null: every token's row of y [T, d] (layer dtype) is set to 0
// (the down-projection then adds the token's rows into it)
cudaError_t launch_route_gate(const moe_config *c, const float *logits_in, float *logits_out,
                              const void *x, const void *w_router, const float *bias,
                              const float *state, float *probs, int32_t *topk_idx, float *topk_gate,
                              int32_t *hist, cudaStream_t s, int nsplit = 1,
                              int64_t split_stride = 0, void *y_zero = nullptr);
// DeepSeek-V3 routing-bias update from a step's counts (one block)
cudaError_t launch_bias_update(const moe_config *c, const int32_t *counts, float *bias, float gamma,
                               cudaStream_t s);
// fp32 logits on CUDA cores for fp32 layers the fused router does not cover
cudaError_t launch_router_f32(const moe_config *c, const float *x, const float *w, const float *bias,
                              float *logits, cudaStream_t s);

// --- permutation (permute.cu) ---------------------------------------------
// hist_ready: the gate already wrote the unit histogram into the workspace
// gather = false: x_perm is not written (the up-projection GEMM gathers the
// rows itself)
cudaError_t launch_permute(const moe_config *c, const WsLayout &L, char *ws, bool hist_ready,
                           const void *x, const int32_t *topk_idx, const float *topk_gate,
                           const float *probs, int32_t *counts, int32_t *offsets, int32_t *tok_rows,
                           int32_t *row_token, float *row_gate, void *x_perm, int32_t *n_dropped,
                           cudaStream_t s, bool gather = true);

// --- tcgen05 grouped GEMM (gemm_sm100.cu) ---------------------------------
enum GemmEpilogue : int {
  kEpiStoreF32 = 0,   // out fp32 = acc (+ bias[col])           (router logits)
  kEpiRelu = 1,       // out bf16 = relu(acc)                    (up-projection, ReLU)
  kEpiSwiglu = 2,     // out bf16 = silu(acc_gate) * acc_up      (gate/up projection)
  kEpiScale = 3,      // out bf16 = row_gate[row] * acc          (down-projection, gated rows)
  // backward
  kEpiPreRelu = 4,    // out bf16 = acc                          (pre-activation a, recomputed)
  kEpiPreSwiglu = 5,  // out bf16 [row][col] = a, [row][N+col] = u  (gate/up pre-activations)
  kEpiDActRelu = 6,   // dh = g*acc; out bf16 = dh * [a > 0]     (a from aux [row][col])
  kEpiDActSwiglu = 7, // dh = g*acc; s = sigmoid(a): out[row][col] = dh u s (1 + a (1 - s)),
                      //   out[row][N+col] = dh a s              (a, u from aux, ld 2N)
  // forward, combine folded into the down-projection
  kEpiScaleAdd = 8,   // out[add_rows[row]] += bf16(row_gate[row] * acc)  (routed rows; a static
                      //   group's row t adds into out[t]); out zeroed beforehand
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
  int64_t out_rows;         // rows of out (token-N kernel: > 0 enables TMA stores of whole boxes)
  const float *row_gate;    // kEpiScale: gate per routed output row
  const float *bias;        // kEpiStoreF32: [N] or null (ignored when ksplit > 1)
  int ksplit;               // kEpiStoreF32, one static group: split K into ksplit parts and
  int64_t split_stride;     //   write part s of the output at out + s * split_stride
  float *sk_part;           // stream-K partial tiles [kSkSlots][kSkSlotFloats] and their
  int *sk_flags;            //   flags [kSkSlots] (zero between launches); null: no stream-K
  int reverse;              // 1: tiles in reverse order (last group first)
  const int32_t *gather_rows;  // non-null: routed A row r is gather_src[gather_rows[r]]
  const void *gather_src;      //   (the row gather done inside the GEMM; bf16 [src_rows, K])
  int64_t src_rows;
  // B stored [K][N] per group (N contiguous; the weights as they are, read
  // MN-major by the tensor cores): group g's K rows start at row g * b_krows
  // of b (k-blocks < b_kb_split) or of b3 (the rest, from k-block 0 of b3)
  int b_mn;
  int b_kb_split;
  int64_t b_krows;
  const void *aux;          // kEpiDAct*: bf16 pre-activations, ld aux_ld
  int64_t aux_ld;
  // kEpiDAct*: dg_part[row * dg_nt + n] = sum over N-tile n's columns of
  // acc * act(a) for routed rows (the gate gradient's pieces); null: none
  float *dg_part;
  int dg_nt;
  const void *aux2;         // kEpiDActSwiglu with dg_part: the forward's bf16 h [row][aux2_ld]
  int64_t aux2_ld;          //   (the gate-gradient pieces take h from there)
  const int32_t *add_rows;  // kEpiScaleAdd: output row of each routed row (row_token)
  // K-grouped mode (weight gradients): group g computes out_g[M, N] =
  // A[M, kseg[g]:kseg[g+1]] . B[N, kseg[g]:kseg[g+1]]^T over the K columns
  // kseg gives (multiples of 64, device array of n_static + 1 entries; one
  // group per static group, n_routed = 0); A is [M, a_rows = Kp], B [N, Kp]
  // (row-major, K contiguous).  fp32 out: row r < split_m of group g at
  // out + (g*split_m + r)*N, rows r >= split_m at out2 + (g*split_m + r - split_m)*N.
  int kgroup;
  int M;
  const int32_t *kseg;
  int split_m;
  void *out2;
  uint32_t *err;
};
cudaError_t launch_grouped_gemm(const GroupedGemm &g, cudaStream_t s);

// The token-N kernel (weights on the MMA's M side, tokens on its N side)
// serves the forward expert GEMMs when the routed groups average fewer rows
// than this (where 256-row tiles would be mostly padding and 128-row tiles
// still a fifth); MOE_TN_MAX_ROWS=0 at build time turns it off.
#ifndef MOE_TN_MAX_ROWS
#define MOE_TN_MAX_ROWS 384
#endif


// --- backward helpers (backward.cu) ----------------------------------------
cudaError_t launch_transpose_bf16(const void *in, void *out, int R, int C, int64_t ld_in,
                                  int64_t ld_out, int batch, int64_t bstride_in,
                                  int64_t bstride_out, int col_off, cudaStream_t s);
cudaError_t launch_transpose_f32_bf16(const float *in, void *out, int R, int C, int Rpad,
                                      int64_t ld_out, cudaStream_t s);
cudaError_t launch_seg_offsets(const int32_t *offsets, int E, int S, int64_t T, int32_t *kseg,
                               cudaStream_t s);
cudaError_t launch_transpose_segments(const void *src, int64_t ld, const int32_t *map,
                                      const float *scale, int64_t shared_base, int64_t shared_stride,
                                      int64_t shared_len, int64_t src_rows, const int32_t *offsets,
                                      const int32_t *kseg, int E, int G, int C, int64_t kp_max,
                                      void *out, uint32_t *err, cudaStream_t s);
cudaError_t launch_gather_bf16_rows(const void *src, void *dst, const int32_t *map,
                                    const int32_t *offsets, int E, int64_t src_rows, int d,
                                    int64_t max_rows, uint32_t *err, cudaStream_t s);
cudaError_t launch_gate_grad(const float *dg_part, int nt, const int32_t *offsets, int E,
                             int64_t max_rows, float *dgate, cudaStream_t s);
cudaError_t launch_router_grad(const moe_config *c, const float *probs, const int32_t *topk_idx,
                               const int32_t *tok_rows, const float *dgate, const float *state,
                               float *dl, cudaStream_t s);
cudaError_t launch_bias_grad(const float *dl, int64_t T, int E, float *dbias, cudaStream_t s);
cudaError_t launch_dx_finish(const moe_config *c, int64_t rows_cap, const float *dx_rows,
                             const int32_t *tok_rows, const float *dx_router, float *dx,
                             cudaStream_t s);
cudaError_t launch_pad_f32_bf16(const float *in, void *out, int64_t R, int C, int Cp,
                                cudaStream_t s);
// K parts of the bf16 router GEMM: enough CTAs to fill the GPU, >= 4 k-blocks each
inline int router_ksplit(const moe_config *c) {
  const int64_t mtiles = (c->T + 127) / 128;
  const int kb = c->d_model / 64;
  int ks = (int)(148 / mtiles);
  if (ks > 4) ks = 4;
  while (ks > 1 && kb / ks < 4) --ks;
  return ks < 1 ? 1 : ks;
}
// --- tensor maps (gemm_sm100.cu) ---------------------------------------------
// TMA descriptor of a bf16 matrix [outer][inner] (inner contiguous) read in
// boxes of box_outer rows x 64 columns with the 128-byte swizzle; false when
// the driver refuses it.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
              uint32_t box_outer);
int device_sms();

// --- router GEMM with the gate in its epilogue (router_tc.cu) ---------------
// true when moe_route / moe_forward run the bf16 router through it
bool router_tc_used(const moe_config *c);
// logits_out may be null (not written); topk_idx null: expert choice
// (probabilities only); hist null: no unit histogram; y_zero as for
// launch_route_gate
cudaError_t launch_router_tc(const moe_config *c, const void *x, const void *w_router,
                             const float *bias, const float *state, float *logits_out, float *probs,
                             int32_t *topk_idx, float *topk_gate, int32_t *hist, void *y_zero,
                             uint32_t *err, cudaStream_t s);

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
