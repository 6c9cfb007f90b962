/*
 * moe.h - C ABI of libmoe.so: the forward pass of a sparse Mixture-of-Experts
 * FFN layer on one NVIDIA B200 (sm_100a), and its backward pass (moe_backward).
 *
 * The layer, in five steps (all arithmetic runs in this library's CUDA
 * kernels):
 *   1. router logits  l = x . W_r^T (+ b)
 *        - "大语言模型并行策略（七）：专家并行", section "Mixture of Experts (MoE)":
 *          the router is an FFN plus a softmax layer (read: one bias-free
 *          linear layer over the routed experts; b is an optional fixed bias).
 *   2. softmax gating  p_i = exp(g_i) / sum_j exp(g_j)
 *        - "MoE技术演进", "Adaptive Mixtures of Local Experts", gating equation.
 *   3. selection: token-choice top-k (lower expert index wins ties), optional
 *      group-limited routing, expert capacity with overflow dropped to the
 *      residual, per-expert affinity-based token dropping, shared experts, or
 *      expert choice (each expert takes its top-C tokens)
 *        - "MoE技术演进": selector; GShard section 1 (top-2, capacity C = O(N/E));
 *          DeepSeek-V2 section 3 (device-limited routing) and section 5
 *          (token dropping); DeepSeekMoE section 2 (shared expert isolation).
 *        - LocMoE+ article (机器之心): token-choice vs expert-choice routers.
 *   4. permutation of the kept (token, expert) pairs into expert-contiguous rows
 *        - the single-GPU counterpart of the count-then-fill all-to-all buffers,
 *          "大语言模型并行策略（七）：专家并行", section "MoE 中的 all-to-all 通信".
 *   5. expert FFNs  w_o . ReLU(w_i . x)  (GShard section 3)  or SwiGLU
 *      w_2 . (SiLU(w_1 . x) * (w_3 . x)) with 3 * d_model * d_moe parameters
 *      ("大语言模型并行策略（七）", parameter-count notes), then the
 *      gate-weighted combine  y_t = sum_e G_{t,e} FFN_e(x_t) + sum_s FFN_s(x_t)
 *      (GShard section 3; DeepSeekMoE section 2).  The residual "+ u" of the
 *      DeepSeekMoE equations is left to the caller.
 *
 * Conventions that hold for every entry point:
 *   - Ownership: the caller owns every buffer.  The library allocates no
 *     device memory on any path; scratch lives in the caller's workspace
 *     (moe_query_sizes gives its size).  The one exception is the fixed
 *     array of MOE_PERMUTE_NOALLOC_SCRATCH_BYTES compiled into the library
 *     for moe_permute_noalloc, which every GPU that loads the library holds
 *     until the process exits.  Every tensor pointer is a DEVICE pointer on
 *     the current CUDA device; the structs are host memory.
 *   - Layout: row-major.  x [T, d]; w_router [E, d]; w1, w3 [E+S, f, d];
 *     w2 [E+S, d, f] (each output neuron's weights contiguous along its input
 *     dimension); experts 0..E-1 are routed, E..E+S-1 shared.  Element type
 *     fp32 (MOE_F32) or bf16 (MOE_BF16) for x, weights, x_perm, h, y_rows
 *     and y (the combine sums rows in fp32 and rounds once).  Router logits,
 *     probabilities and gates are always fp32; indices int32.
 *   - Alignment: tensor pointers 16-byte aligned, the workspace 256-byte
 *     aligned.  Limits of this build (else MOE_ERR_UNSUPPORTED): E <= 256,
 *     S <= 8, k <= 8, n_groups <= 32, topk_groups <= 8, T*k and E*C below
 *     2^31; bf16: d and f multiples of 64; fp32: d a multiple of 4.
 *   - Streams: every call is asynchronous on `stream` (a cudaStream_t) and
 *     never synchronises with the host, except moe_check_device_errors.
 *   - Errors: arguments are validated on the host before any launch; nothing
 *     is launched when a call returns an error.  Launch failures return
 *     MOE_ERR_CUDA.  Kernels never trap: a device-side wait that exceeds its
 *     time limit sets a bit in the error word at the start of the workspace
 *     and the kernel returns; moe_check_device_errors reads it.
 *   - Reentrancy: calls may run concurrently on different streams with
 *     different workspaces.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size or option               */
  MOE_ERR_UNSUPPORTED = 2,  /* valid layer, but outside this build's limits   */
  MOE_ERR_WORKSPACE = 3,    /* workspace smaller than moe_query_sizes says    */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed    */
  MOE_ERR_DEVICE_CHECK = 5, /* a kernel reported a bad index in its checks    */
  MOE_ERR_TIMEOUT = 6       /* a kernel's bounded wait ran out                */
} moe_status;

typedef enum moe_dtype { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum moe_act { MOE_ACT_RELU = 0, MOE_ACT_SWIGLU = 1 } moe_act;
typedef enum moe_mode { MOE_TOKEN_CHOICE = 0, MOE_EXPERT_CHOICE = 1 } moe_mode;
/* What token-choice top-k selects on ("MoE技术演进"):
 *   SOFTMAX  key = logit g, gate = p (the plain selector);
 *   BIAS     DeepSeek-V3 item 1, auxiliary-loss-free balancing: key = p + b_e
 *            (one fp32 add; the affinity s read as p), gate = p + b_e as the
 *            printed formula gives it; b = route_state [E];
 *   LOAD     interview question Q3 item 3, load-aware top-k: key = g +
 *            route_alpha * (1 - u_e) (fp32: o = alpha * (1 - u), key = g + o),
 *            gate = p; u = route_state [E], the experts' utilisation. */
typedef enum moe_route_rule { MOE_ROUTE_SOFTMAX = 0, MOE_ROUTE_BIAS = 1, MOE_ROUTE_LOAD = 2 } moe_route_rule;

/* The layer.  Capacity, keep-fraction and expert choice are exclusive.
 *
 * Expert capacity (GShard section 1 of "MoE技术演进": each expert takes at
 * most C = O(N/E) tokens, the overflow passes to the residual; with local
 * group dispatching the capacity of a group of N/G tokens, 2N/(G*E) for
 * top-2 at factor 1).  The library derives C from the factor:
 *     C = ceil(capacity_factor * k * T / E)          (one group)
 *     C = ceil(capacity_factor * k * (T / G) / E)    (local_groups G > 1, per group)
 * evaluated exactly for the fp32 value given (no rounding before the
 * ceiling; 0.1f is slightly above 0.1, so 0.1f * 10 gives 2) and clamped to
 * the group's token count (an expert receives at most one assignment per
 * token).  moe_sizes.capacity reports C. */
typedef struct moe_config {
  int64_t T;           /* tokens in this call (>= 1)                                */
  int32_t d_model;     /* d                                                         */
  int32_t E;           /* routed experts (>= 1)                                     */
  int32_t S;           /* shared experts, gate 1 for every token (>= 0)             */
  int32_t k;           /* experts per token, token choice (1 <= k <= E)             */
  int32_t d_ff;        /* expert hidden size f (d_ff, or d_moe for SwiGLU)          */
  float capacity_factor; /* token choice: expert capacity factor cf; <= 0 unlimited  */
  int32_t keep_num;    /* token choice: expert e keeps ceil(n_e*num/den) of its n_e */
  int32_t keep_den;    /*   assignments by affinity; den = 0: keep all              */
  int32_t ec_capacity; /* expert choice: tokens per expert C (1 <= C <= T)          */
  int32_t n_groups;    /* group-limited routing: E/n_groups contiguous experts per  */
  int32_t topk_groups; /*   group, keep topk_groups groups per token; 0,0 = off     */
  int32_t renormalize; /* 1: gate = p / (sum of the selected p)                     */
  int32_t act;         /* moe_act                                                   */
  int32_t mode;        /* moe_mode                                                  */
  int32_t dtype;       /* moe_dtype                                                 */
  int32_t route_rule;  /* moe_route_rule (token choice; SOFTMAX in expert choice)   */
  float route_alpha;   /* MOE_ROUTE_LOAD: alpha                                     */
  int32_t local_groups;/* GShard local groups G (0 or 1: one group): T/G contiguous  */
                       /*   tokens per group, each dispatching on its own with C    */
                       /*   rows per expert; needs capacity_factor > 0, T % G == 0  */
                       /*   and (T/G) % 32 == 0                                     */
  int32_t reserved;    /* 0                                                         */
} moe_config;

/* Buffer sizes of one configuration. */
typedef struct moe_sizes {
  int64_t rows_cap;        /* routed rows, worst case: T*k (token choice), E*C (expert choice) */
  int64_t rows_total;      /* rows of h and y_rows: rows_cap + S*T                              */
  int64_t tok_rows_len;    /* entries of tok_rows: T*k (token choice) or E*T (expert choice)     */
  size_t step_workspace;   /* bytes of workspace the step entry points need                     */
  size_t workspace;        /* bytes of workspace moe_forward needs (>= step_workspace)          */
  int64_t capacity;        /* token choice: expert capacity C the library derived from          */
                           /*   capacity_factor (per local group); 0: unlimited or not token    */
                           /*   choice.  Expert choice's C is ec_capacity                       */
  size_t permute_workspace;/* bytes of scratch moe_permute uses (<= step_workspace): what       */
                           /*   moe_permute_noalloc needs from its fixed array                  */
  size_t host_workspace;   /* bytes of workspace moe_forward_host needs (>= workspace): the     */
                           /*   forward's, plus device staging rows for x and y                  */
} moe_sizes;

/* Sizes of every buffer for `cfg`.  Validates cfg: returns MOE_ERR_INVALID_ARG
 * or MOE_ERR_UNSUPPORTED exactly when the compute entry points would. */
MOE_API moe_status moe_query_sizes(const moe_config *cfg, moe_sizes *out);

/* Steps 1-3a: router logits, softmax, token-choice top-k.
 *   x [T, d], w_router [E, d] (cfg dtype); bias [E] fp32 or NULL (added to
 *   the logits); route_state [E] fp32: the routing bias b (MOE_ROUTE_BIAS) or
 *   the utilisation u (MOE_ROUTE_LOAD), NULL with MOE_ROUTE_SOFTMAX.
 *   out: logits [T, E], probs [T, E] fp32;
 *        topk_idx [T, k] int32 in rank order, topk_gate [T, k] fp32
 *        (both ignored and may be NULL in expert-choice mode).
 *   Top-k keys are those of cfg->route_rule (the fp32 logits by default):
 *   strictly larger first, lower expert index on ties; with group limits
 *   only the topk_groups groups with the largest maximum key (lower group on
 *   ties) compete.  p is computed in a fixed
 *   fp32 recipe (own exp, sequential ascending-expert sum, IEEE division) so
 *   that it is reproducible bit for bit.
 *   ws: workspace of at least step_workspace bytes. */
MOE_API moe_status moe_route(const moe_config *cfg, const void *x, const void *w_router, const float *bias,
                     const float *route_state, float *logits, float *probs, int32_t *topk_idx,
                     float *topk_gate, void *ws, size_t ws_bytes, moe_stream_t stream);

/* Steps 2-3a from given fp32 logits [T, E] (the same arithmetic moe_route
 * applies after its router GEMM).  Outputs as moe_route. */
MOE_API moe_status moe_gate(const moe_config *cfg, const float *logits, const float *route_state,
                    float *probs, int32_t *topk_idx, float *topk_gate, void *ws, size_t ws_bytes,
                    moe_stream_t stream);

/* DeepSeek-V3's per-step routing-bias update ("MoE技术演进", DeepSeek-V3
 * item 1): with counts [E] from a step (assignments per expert, as
 * moe_permute / moe_forward report them), an expert above the mean load
 * T*k/E lowers its bias by gamma, one below raises it by gamma, one exactly
 * at the mean keeps it.  The load test is exact integer arithmetic
 * (counts[e]*E against T*k); the step one fp32 add.  route_bias [E] fp32 is
 * updated in place.  Token choice only. */
MOE_API moe_status moe_route_bias_update(const moe_config *cfg, const int32_t *counts, float *route_bias,
                                         float gamma, moe_stream_t stream);

/* Steps 3b-4: capacity / keep-fraction / expert choice, then permutation.
 *   in : x [T, d]; token choice: topk_idx, topk_gate [T, k] (+ probs [T, E]
 *        for keep-fraction); expert choice: probs [T, E] (topk_* may be NULL).
 *   out: counts [E]    assignments per expert before drops (expert choice: C)
 *        offsets [E+1] exclusive scan of the rows each expert keeps
 *        tok_rows      token choice [T, k]: row of (t, j), -1 when dropped;
 *                      expert choice [E, T]: row of (e, t), -1 when not taken
 *        row_token [rows_cap], row_gate [rows_cap]: token and gate of each row
 *                      (entries >= offsets[E] are unspecified)
 *        x_perm [rows_cap, d]: x_perm[r] = x[row_token[r]] byte for byte
 *        n_dropped [1] token-choice assignments dropped (0 in expert choice)
 *   Token choice keeps rows of an expert in priority order q = j*T + t; with a
 *   capacity C the assignment of priority q survives iff fewer than C earlier
 *   ones went to its expert.  Keep-fraction keeps, per expert, the
 *   ceil(n_e*num/den) assignments with the largest p[t, e] (lower t on ties).
 *   Expert choice: expert e takes the C tokens with the largest p[t, e]
 *   (lower t on ties), in ascending t; rows e*C .. e*C+C-1.
 *   All integer outputs are deterministic and bit-exact. */
MOE_API moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                       const float *topk_gate, const float *probs, int32_t *counts, int32_t *offsets,
                       int32_t *tok_rows, int32_t *row_token, float *row_gate, void *x_perm,
                       int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute without a workspace argument.  The paper has no counterpart:
 * this entry point is for callers that cannot allocate device memory (a
 * plugin in a host program that is handed only its input and output buffers,
 * or a process that must keep a fixed device footprint once started) and so
 * cannot provide moe_permute's workspace.
 *   Arguments, outputs and results are those of moe_permute.
 *   Scratch: a fixed array of MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (8 MiB) compiled
 *   into the library, held by every GPU that loads the library until the
 *   process exits.  The permutation's scratch (moe_sizes.permute_workspace:
 *   the control block, the unit histograms and their block sums, the count
 *   and row offsets, and the keep-fraction list or the transposed
 *   probabilities of expert choice) must fit in it, else the call returns
 *   MOE_ERR_WORKSPACE before any launch.  It calls no cudaMalloc, cudaFree or
 *   allocating routine.
 *   Set-up: the first call on each device looks up the array's device address
 *   with that device current; make that first call before any stream capture.
 *   Later calls look it up again whenever `stream` is not capturing (so a
 *   device reset, which reloads the library's device code, is picked up) and
 *   reuse the last address while it is.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents (each call clears what must start at zero).  Calls that
 *   overlap on the GPU -- other streams or threads -- race on it and give wrong
 *   results; serialise them.
 *   Errors: the array's error word is cleared at the start of each call; bad
 *   expert indices are still skipped, but their report cannot be read here
 *   (moe_permute with a workspace and moe_check_device_errors shows it). */
#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
MOE_API moe_status moe_permute_noalloc(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                                       const float *topk_gate, const float *probs, int32_t *counts,
                                       int32_t *offsets, int32_t *tok_rows, int32_t *row_token,
                                       float *row_gate, void *x_perm, int32_t *n_dropped,
                                       moe_stream_t stream);

/* Step 5a-5b: the grouped expert FFNs.
 *   in : x [T, d] (input of the shared experts), x_perm [rows_cap, d],
 *        offsets [E+1], row_gate [rows_cap], w1, w3 (SwiGLU; NULL for ReLU), w2.
 *   out: h [rows_total, f]  activations, layer dtype (scratch the caller may read);
 *        y_rows [rows_total, d], layer dtype: routed row r = row_gate[r] * FFN_e(x_perm[r]);
 *        shared expert s, token t at row rows_cap + s*T + t = FFN_{E+s}(x[t]).
 *   bf16: tcgen05 tensor cores, bf16 operands, fp32 accumulation, h rounded
 *   to bf16.  fp32: CUDA-core fp32 arithmetic. */
MOE_API moe_status moe_expert_ffn(const moe_config *cfg, const void *x, const void *x_perm,
                          const int32_t *offsets, const float *row_gate, const void *w1,
                          const void *w3, const void *w2, void *h, void *y_rows, void *ws,
                          size_t ws_bytes, moe_stream_t stream);

/* Step 5c: y[t] = sum of t's routed rows (layer dtype; token choice: in k-rank order;
 * expert choice: ascending expert) + its shared rows, fp32 accumulation,
 * rounded once to the layer dtype.  A token with no kept row and no shared
 * expert gets 0. */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_rows, const int32_t *tok_rows, void *y,
                       moe_stream_t stream);

/* Steps 1-5 in one call; intermediates live in the workspace (at least
 * `workspace` bytes).  counts_out [E] (optional, may be NULL) receives the
 * per-expert assignment counts.  Same result as moe_route, moe_permute,
 * moe_expert_ffn and moe_combine in sequence, bit for bit.  bf16 token
 * choice with k + S <= 2 (at most two rows a token) folds the combine into
 * the expert FFN: y is zeroed by the routing kernel and each gated row is
 * added into its token's row by the down-projection (two bf16 additions onto
 * 0, which commute), so the workspace holds no y_rows afterwards and no
 * combine kernel runs.  y [T, d] must not overlap x (MOE_ERR_INVALID_ARG). */
MOE_API moe_status moe_forward(const moe_config *cfg, const void *x, const void *w_router,
                       const float *bias, const float *route_state, const void *w1, const void *w3,
                       const void *w2, void *y, int32_t *counts_out, void *ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_forward on HOST buffers: x_host [T, d] is copied into the workspace,
 * the layer runs as moe_forward does, and y comes back to y_host [T, d] (both
 * in the layer dtype; page-locked host memory lets the copies run
 * asynchronously at full speed).  Everything is queued without a host sync:
 * the host buffers must stay untouched until y_host's copy has completed
 * (synchronise `copy_out`, or `stream` when copy_out is NULL).
 *   stream: the forward's kernels.  copy_in / copy_out: streams for the
 *   host-to-device and device-to-host copies (NULL: `stream`).  With two
 *   copy streams and two workspaces used in turn, the copies of one call
 *   overlap the forward of the call before and after it; the forwards
 *   themselves stay in order on `stream`.
 *   The library orders the calls that share a workspace itself: a call's
 *   input copy waits for the previous forward on that workspace, its forward
 *   for the previous output copy.  For that it keeps three CUDA events per
 *   workspace used here (host objects, no device memory) until the process
 *   exits.
 *   ws: at least moe_sizes.host_workspace bytes.  counts_out as moe_forward
 *   (device memory or NULL).  Errors as moe_forward; MOE_ERR_INVALID_ARG for
 *   a NULL host buffer. */
MOE_API moe_status moe_forward_host(const moe_config *cfg, const void *x_host, const void *w_router,
                                    const float *bias, const float *route_state, const void *w1,
                                    const void *w3, const void *w2, void *y_host,
                                    int32_t *counts_out, void *ws, size_t ws_bytes,
                                    moe_stream_t stream, moe_stream_t copy_in,
                                    moe_stream_t copy_out);

/* moe_forward that also records caller-created CUDA events on `stream` at
 * its phase boundaries: events[0] before step 1, [1] after steps 1-3a
 * (routing), [2] after 3b-4 (permutation), [3] after 5a-5b (expert FFNs),
 * [4] after 5c (combine).  events: array of 5 cudaEvent_t handles (entries may
 * be NULL).  Same launches and results as moe_forward. */
MOE_API moe_status moe_forward_timed(const moe_config *cfg, const void *x, const void *w_router,
                                     const float *bias, const float *route_state, const void *w1,
                                     const void *w3, const void *w2, void *y, int32_t *counts_out,
                                     void *ws, size_t ws_bytes, void *const *events,
                                     moe_stream_t stream);

/* Backward pass (training) of the forward that last ran on `ws`: gradients
 * of L = sum(dy * y) ("MoE技术演进": GShard, DeepSeekMoE and DeepSeek-V2/V3
 * are trained this way; the gate is the softmax gating network of "Adaptive
 * Mixtures of Local Experts").  The routing decisions of that forward (top-k,
 * capacity drops, keep-fraction, expert choice, local groups) are held fixed;
 * gradient reaches the experts through every kept row and the router through
 * the gate of each kept row (G = p, p / sum of the selected p when
 * renormalised, p + b under MOE_ROUTE_BIAS).  bf16 layers only
 * (MOE_ERR_UNSUPPORTED for fp32).
 *   in : the forward's x, w_router, bias, route_state, w1, w3, w2 and its
 *        workspace ws (unchanged since moe_forward: the routing, x_perm and h
 *        it holds are read); dy [T, d] bf16.
 *   out: dx [T, d], dw_router [E, d], dbias [E] (NULL when bias is NULL),
 *        dw1 [E+S, f, d], dw3 [E+S, f, d] (SwiGLU; NULL for ReLU),
 *        dw2 [E+S, d, f]: fp32, overwritten.
 *   bws: scratch of at least moe_query_backward_size bytes (256-byte aligned).
 *   Arithmetic: bf16 tensor-core contractions with fp32 accumulation; the
 *   recomputed pre-activations, dA / dU and the transposed operands are
 *   rounded to bf16; gate and router gradients in fp32 (a gate's gradient
 *   <dy, FFN_e(x)> is taken as <dy W2_e, act(a)> inside the dA GEMM). */
MOE_API moe_status moe_query_backward_size(const moe_config *cfg, size_t *bytes);
MOE_API moe_status moe_backward(const moe_config *cfg, const void *x, const void *w_router,
                                const float *bias, const float *route_state, const void *w1,
                                const void *w3, const void *w2, const void *dy, float *dx,
                                float *dw_router, float *dbias, float *dw1, float *dw3, float *dw2,
                                const void *ws, size_t ws_bytes, void *bws, size_t bws_bytes,
                                moe_stream_t stream);

/* Waits for `stream`, then reads and clears the workspace's device error
 * word.  Returns MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_CHECK; *flags (if
 * not NULL) receives the raw bits.  After an error it also clears the rest
 * of the workspace's 4 KiB control block (the GEMMs' stream-K ready flags,
 * which a timed-out launch can leave set).  This is the only call that
 * blocks. */
MOE_API moe_status moe_check_device_errors(void *ws, size_t ws_bytes, moe_stream_t stream, uint32_t *flags);

/* Fill `ws` with the bytes the library expects in a fresh workspace: the
 * 4 KiB control block at its start (error word, the GEMMs' stream-K ready
 * flags) cleared.  Call once after allocating a workspace (a zero-filled
 * allocation needs no call).  Every launch leaves the flags at zero unless
 * it reports an error. */
MOE_API moe_status moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream);

/* Set the time limit of every device-side wait of the launches that use
 * `ws` (bytes 8-15 of its control block): limit_ns nanoseconds, 0 for the
 * default of 2 s.  A wait that runs out sets the timeout bit of the error
 * word and its kernel returns early (its outputs are then incomplete);
 * moe_check_device_errors reports MOE_ERR_TIMEOUT, and clears the control
 * block, which restores the default.  The drains that let a timed-out
 * kernel's copies land always take the default.  Asynchronous on `stream`
 * (a copy from host memory).  Meant for failure detection: a short limit
 * turns a wait that can never finish into an error status within that
 * time. */
MOE_API moe_status moe_workspace_set_wait_limit(void *ws, size_t ws_bytes, uint64_t limit_ns,
                                                moe_stream_t stream);

/* Static text for a status code. */
MOE_API const char *moe_status_string(moe_status s);

/* Number of kernels the library has launched since it was loaded, counted
 * over all threads and devices at each successful launch (host-side
 * counter; touches no CUDA state, so it works without a GPU).  The
 * difference across a region of calls is the number of kernels those calls
 * launched. */
MOE_API uint64_t moe_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
